"""Sparse MLA over a block-table paged latent cache (bf16 or fp8 E4M3) on the GPU.

The same rows stored in pages at scattered places must give the contiguous
call's results bit for bit (the kernels differ only in the row lookup); ids on
missing pages must be ignored as the oracle ignores them. Unused pages hold NaN,
so a read of a wrong row shows.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import assert_mla_close, dev_bits, device_status_clean, mla_value_bound
from sparse_attention_indexer_head_b200 import workloads as W

pytestmark = pytest.mark.gpu

NAN_BF16 = 0x7FC0


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_indexer_head_b200 import build
    build.build()
    from sparse_attention_indexer_head_b200 import binding
    binding.dsa_device_status(reset=True)
    return binding


def _paginate(wl, page, spare, seed, drop=()):
    """Scatter each request's rows over pages of a pool; returns (pool, table, seq_len).

    Pages listed in `drop` as (request, page index) get block -1 (missing)."""
    rng = np.random.default_rng(seed)
    lengths = [int(t) for t in np.diff(wl.req_start)]
    n_pages = [(t + page - 1) // page for t in lengths]
    total = sum(n_pages) + spare
    perm = rng.permutation(total)
    pool = np.full((total * page, wl.kv.shape[1]), NAN_BF16, np.uint16)
    max_blocks = max(1, max(n_pages)) + 1
    table = np.full((wl.B, max_blocks), -1, np.int32)
    k = 0
    for b, T in enumerate(lengths):
        for pi in range(n_pages[b]):
            blk = int(perm[k])
            k += 1
            if (b, pi) in drop:
                continue
            table[b, pi] = blk
            rows = wl.kv[wl.req_start[b] + pi * page: wl.req_start[b] + min(T, (pi + 1) * page)]
            pool[blk * page: blk * page + len(rows)] = rows
    return pool, table, np.asarray(lengths, np.int32)


def _paged_call(B, step, pool, table, seq_len, page):
    g, t = step.g, step.t
    out = torch.empty_like(step.out)
    lse = torch.empty_like(step.lse)
    ws = torch.empty(max(16, B.dsa_sparse_mla_workspace_size(g.Q, g.hm, g.W)), dtype=torch.uint8,
                     device="cuda")
    B.dsa_sparse_mla_decode_paged(
        t["q_mla"], dev_bits(pool), pool.shape[0], torch.from_numpy(table).cuda(), table.shape[1],
        page, torch.from_numpy(seq_len).cuda(), t["q_req"], step.token_ids, g.Q, g.B, g.hm, g.W,
        512, 0, g.sm_scale, out, lse, ws, ws.numel())
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy().view(np.uint16), lse.cpu().numpy()


def _workload(name):
    if name == "split4":
        # 32 decode queries: each query's ids split 4 ways, merged by the combine
        lengths = [600 + 37 * i for i in range(32)]
        return W.build("split4", lengths=lengths, pads=[i % 5 for i in range(32)], kpool=4,
                       max_pools=(max(lengths) + 3) // 4, select_k=512, hm=64,
                       q_req=list(range(32)), q_pos=[t - 1 for t in lengths], seed=17)
    return W.make(name)


@pytest.mark.parametrize("name,page", [("tiny", 16), ("tiny", 7), ("tiny", 1), ("batched", 64),
                                       ("split4", 32)])
def test_paged_equals_contiguous(B, name, page):
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    wl = _workload(name)
    step = DecodeStep(wl)
    step.run()
    torch.cuda.synchronize()
    g = step.outputs_numpy()
    pool, table, seq_len = _paginate(wl, page, spare=3, seed=page)
    out, lse = _paged_call(B, step, pool, table, seq_len, page)
    np.testing.assert_array_equal(out, g["out"])
    np.testing.assert_array_equal(lse, g["lse"])
    device_status_clean(B)


def test_paged_missing_pages_and_short_sequences(B):
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    lengths = [300, 129, 64]
    wl = W.build("paged edges", lengths=lengths, pads=[0, 3, 0], kpool=4, max_pools=80,
                 select_k=32, hm=16, q_req=[0, 1, 2, 0], q_pos=[299, 128, 63, 150], seed=8)
    step = DecodeStep(wl)
    step.run()
    torch.cuda.synchronize()
    g = step.outputs_numpy()
    page = 16
    drop = {(0, 3), (1, 0), (2, 3)}                 # three pages missing from the table
    pool, table, seq_len = _paginate(wl, page, spare=2, seed=1, drop=drop)
    seq_len[2] = 40                                 # request 2 shorter than its cached rows
    out, lse = _paged_call(B, step, pool, table, seq_len, page)
    ref_out, ref_lse = O.sparse_mla_paged(wl.q_mla, pool, table, page, seq_len, wl.q_req,
                                          g["token_ids"], wl.sm_scale)
    ids = g["token_ids"].copy()
    vb = mla_value_bound(wl.kv, wl.req_start, wl.q_req, ids)
    assert_mla_close(out, ref_out, lse, ref_lse, vbound=vb)
    assert np.isfinite(W.bf16_bits_to_f32(out)).all()    # no NaN page was read
    device_status_clean(B)


def _fp8_cache(wl, scale):
    """The workload's latent cache quantised to E4M3 codes for the given scale (input
    generation: torch's float8_e4m3fn cast of kv / scale)."""
    x = torch.from_numpy(W.bf16_bits_to_f32(wl.kv)) / scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _paged_call_fp8(B, step, pool8, scale, table, seq_len, page):
    g, t = step.g, step.t
    out = torch.empty_like(step.out)
    lse = torch.empty_like(step.lse)
    ws = torch.empty(max(16, B.dsa_sparse_mla_workspace_size(g.Q, g.hm, g.W)), dtype=torch.uint8,
                     device="cuda")
    B.dsa_sparse_mla_decode_paged_fp8(
        t["q_mla"], torch.from_numpy(pool8).cuda(), scale, pool8.shape[0],
        torch.from_numpy(table).cuda(), table.shape[1], page, torch.from_numpy(seq_len).cuda(),
        t["q_req"], step.token_ids, g.Q, g.B, g.hm, g.W, 512, 0, g.sm_scale, out, lse, ws,
        ws.numel())
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy().view(np.uint16), lse.cpu().numpy()


@pytest.mark.parametrize("name,page", [("tiny", 16), ("batched", 64), ("split4", 32)])
def test_paged_fp8_against_oracle_and_bf16(B, name, page):
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    wl = _workload(name)
    rng = np.random.default_rng(31)
    kv8 = _fp8_cache(wl, 0.37)
    step = DecodeStep(wl)
    step.run()
    torch.cuda.synchronize()
    ids = step.token_ids.cpu().numpy()
    # the same fp8 rows scattered over pages (unused pages hold NaN codes)
    lengths = [int(x) for x in np.diff(wl.req_start)]
    n_pages = [(t + page - 1) // page for t in lengths]
    total = sum(n_pages) + 2
    perm = rng.permutation(total)
    pool8 = np.full((total * page, 512), 0x7F, np.uint8)
    table = np.full((wl.B, max(n_pages) + 1), -1, np.int32)
    k = 0
    for b, T in enumerate(lengths):
        for pi in range(n_pages[b]):
            blk = int(perm[k]); k += 1
            table[b, pi] = blk
            rows = kv8[wl.req_start[b] + pi * page: wl.req_start[b] + min(T, (pi + 1) * page)]
            pool8[blk * page: blk * page + len(rows)] = rows
    seq_len = np.asarray(lengths, np.int32)
    # a scale that is not a power of two: against the oracle
    out, lse = _paged_call_fp8(B, step, pool8, 0.37, table, seq_len, page)
    ref_out, ref_lse = O.sparse_mla_fp8(wl.q_mla, kv8, 0.37, wl.req_start, wl.q_req, ids,
                                        wl.sm_scale)
    dec = np.array([O.f64_from_e4m3(c) for c in range(256)])
    vb = mla_value_bound(0.37 * dec[kv8], wl.req_start, wl.q_req, ids)
    assert_mla_close(out, ref_out, lse, ref_lse, vbound=vb)
    assert np.isfinite(W.bf16_bits_to_f32(out)).all()
    # a power-of-two scale: bit-identical to the bf16 kernel on the decoded, scaled cache
    kv_b = W.f32_to_bf16_bits((0.5 * dec[kv8]).astype(np.float32))
    pool_b = np.zeros((pool8.shape[0], 512), np.uint16)
    used = table[table >= 0]
    for b, T in enumerate(lengths):
        for pi in range(n_pages[b]):
            blk = table[b, pi]
            rows = kv_b[wl.req_start[b] + pi * page: wl.req_start[b] + min(T, (pi + 1) * page)]
            pool_b[blk * page: blk * page + len(rows)] = rows
    out8, lse8 = _paged_call_fp8(B, step, pool8, 0.5, table, seq_len, page)
    outb, lseb = _paged_call(B, step, pool_b, table, seq_len, page)
    np.testing.assert_array_equal(out8, outb)
    np.testing.assert_array_equal(lse8, lseb)
    assert used.size == sum(n_pages)
    device_status_clean(B)


def test_split4_workload_plan(B):
    """The 32-query case above: 4 splits a query (128 CTAs), merged by the combine."""
    assert B.dsa_sparse_mla_launch_count(32, 64, 2048) == 2
    assert B.dsa_sparse_mla_workspace_size(32, 64, 2048) == 32 * 4 * 64 * (1024 + 8)
