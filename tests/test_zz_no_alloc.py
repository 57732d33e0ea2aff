"""The allocation-free sparse-MLA entry point against the regular one.

dsa_sparse_mla_decode_noalloc serves callers that cannot allocate device memory
where they run the MLA (everything they use was reserved before the step
started), so it takes no workspace and uses the library's own static scratch.
Its results must match dsa_sparse_mla_decode, which uses a caller workspace.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test. It passes alone in a fresh
process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import assert_mla_close, dev_bits, host_bits, mla_value_bound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    return binding


def _case(seed=7, Q=16, lengths=8192, Wd=2048, hm=64):
    rng = np.random.default_rng(seed)
    T = Q * lengths
    rs = (np.arange(Q + 1) * lengths).astype(np.int32)
    kv = (rng.standard_normal((T, 512)).astype(np.float32))
    q = (rng.standard_normal((Q, hm, 512)).astype(np.float32))
    from sparse_attention_indexer_head_b200.workloads import f32_to_bf16_bits
    ids = np.stack([rng.choice(lengths, Wd, replace=False) for _ in range(Q)]).astype(np.int32)
    ids[:, -37:] = -1                      # a sentinel tail, as top-k emits it
    return f32_to_bf16_bits(q), f32_to_bf16_bits(kv), rs, np.arange(Q, dtype=np.int32), ids


@pytest.mark.parametrize("Q,Wd", [(2, 8192), (16, 2048)])
def test_noalloc_matches_workspace_entry_point(B, Q, Wd):
    # 2 queries of 8192 ids: 43 splits each; 16 queries of 2048: 9 splits each; both
    # merged through the scratch
    q, kv, rs, q_req, ids = _case(Q=Q, Wd=Wd)
    Q, hm, _ = q.shape
    scale = float(1 / np.sqrt(512))
    need = B.dsa_sparse_mla_workspace_size(Q, hm, Wd)
    assert 0 < need <= B.DSA_NOALLOC_SCRATCH_BYTES
    assert B.dsa_sparse_mla_launch_count(Q, hm, Wd) == 2          # the scratch is used
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    dq, dkv, drs, dqr, dids = dev_bits(q), dev_bits(kv), d(rs), d(q_req), d(ids)

    ref_out = torch.empty(Q, hm, 512, dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty(Q, hm, dtype=torch.float32, device="cuda")
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    B.dsa_sparse_mla_decode(dq, dkv, kv.shape[0], drs, dqr, dids, Q, Q, hm, Wd, 512, 0, scale,
                            ref_out, ref_lse, ws, need)
    torch.cuda.synchronize()
    r_out, r_lse = host_bits(ref_out), ref_lse.cpu().numpy()
    vb = mla_value_bound(kv, rs, q_req, ids)

    for _ in range(2):                      # two calls in a row share the one scratch area
        out = torch.full((Q, hm, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((Q, hm), float("nan"), dtype=torch.float32, device="cuda")
        B.dsa_sparse_mla_decode_noalloc(dq, dkv, kv.shape[0], drs, dqr, dids, Q, Q, hm, Wd, 512,
                                        0, scale, out, lse)
        torch.cuda.synchronize()
        # same kernels, same split order: bit-identical
        np.testing.assert_array_equal(host_bits(out), r_out)
        np.testing.assert_array_equal(lse.cpu().numpy(), r_lse)

    # and both agree with the oracle on one query
    o_out, o_lse = O.sparse_mla(q[:1], kv, rs, q_req[:1], ids[:1], scale)
    assert_mla_close(r_out[:1], o_out, r_lse[:1], o_lse, vbound=vb[:1])
    assert B.dsa_device_status(reset=True) == 0
