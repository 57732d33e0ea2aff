"""always_select_tail on the GPU: dsa_topk_expand_tail and the MLA over the
wider index row, against the oracle (top-k and tail slots bit-exact, MLA within
the bf16 bounds)."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import assert_mla_close, device_status_clean, mla_value_bound
from sparse_attention_indexer_head_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    binding.dsa_device_status(reset=True)
    return binding


def _run_tail(wl):
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    step = DecodeStep(wl, always_select_tail=True)
    step.token_ids.fill_(0x7F7F7F7F)            # every slot must be written
    step.run()
    torch.cuda.synchronize()
    return step, step.outputs_numpy()


def _check(wl, g):
    K, kp = wl.select_k, wl.kpool
    assert g["token_ids"].shape == (wl.Q, K * kp + kp - 1)
    # top-k and expansion on the GPU's own scores: bit-exact
    top, ids = O.topk_expand(g["scores"], g["cand"], g["pool_idx"], wl.q_req, K)
    np.testing.assert_array_equal(g["top_pools"], top)
    np.testing.assert_array_equal(g["token_ids"][:, :K * kp], ids)
    # tail slots: bit-exact
    tail = O.tail_slots(wl.q_req, wl.q_pos, g["first_valid"], wl.valid, wl.req_start, kp)
    np.testing.assert_array_equal(g["token_ids"][:, K * kp:], tail)
    # no token twice in a row
    for row in g["token_ids"]:
        v = row[row >= 0]
        assert len(np.unique(v)) == len(v)
    # MLA over the whole row
    out, lse = O.sparse_mla(wl.q_mla, wl.kv, wl.req_start, wl.q_req, g["token_ids"], wl.sm_scale)
    vb = mla_value_bound(wl.kv, wl.req_start, wl.q_req, g["token_ids"])
    return tail, assert_mla_close(g["out"], out, g["lse"], lse, vbound=vb)


@pytest.mark.parametrize("kpool", [2, 3, 4, 8])
def test_tail_slots_ragged_requests(B, kpool):
    lengths = [37, 300, 129, 0, 64, 11]
    pads = [5, 17, 129, 0, 0, 0]                 # request 2 is all padding, 3 is empty
    holes = [37 + 300 - 2]                       # a hole near the end of request 1
    # decode queries at T - 1 plus mid-context queries on every tail length
    q_req, q_pos = [], []
    for b, T in enumerate(lengths):
        q_req.append(b)
        q_pos.append(max(T - 1, 0))
    for off in range(kpool + 1):
        q_req.append(1)
        q_pos.append(150 + off)
    q_req.append(0)
    q_pos.append(2)                              # before request 0's first valid token
    mp = max(1, max((t + kpool - 1) // kpool for t in lengths))
    wl = W.build(f"tail k{kpool}", lengths=lengths, pads=pads, kpool=kpool, max_pools=mp,
                 select_k=8, hm=16, q_req=q_req, q_pos=q_pos, seed=40 + kpool, holes=holes)
    step, g = _run_tail(wl)
    tail, rep = _check(wl, g)
    assert (tail >= 0).any()                     # some query does attend a tail
    assert (tail[-1] == -1).all()
    device_status_clean(B)


def test_tail_on_the_batched_decode_workload(B):
    wl = W.make("batched")
    step, g = _run_tail(wl)
    _, rep = _check(wl, g)
    device_status_clean(B)


def test_tail_with_select_k_zero_writes_only_the_tail(B):
    wl = W.build("tail only", lengths=[30], pads=[0], kpool=4, max_pools=8, select_k=0, hm=16,
                 q_req=[0, 0], q_pos=[29, 26], seed=2)
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    step = DecodeStep(wl, always_select_tail=True)
    step.kpool_compress()
    step.head_gate()
    step.index_scores()
    step.token_ids.fill_(0x7F7F7F7F)
    step.topk_expand()
    torch.cuda.synchronize()
    ids = step.token_ids.cpu().numpy()
    np.testing.assert_array_equal(ids, [[28, 29, -1], [24, 25, 26]])
    device_status_clean(B)
