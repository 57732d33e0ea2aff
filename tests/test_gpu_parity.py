"""GPU path (through the C ABI) against the CPU oracle, stage by stage.

Every oracle stage is fed the GPU's own inputs to that stage, so rounding in an
earlier stage cannot leak into a later comparison; an end-to-end comparison
from raw inputs follows. Workloads are the seeded synthetic configurations
(tiny, batched, ragged, long-context, prefill) plus edge cases.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import (assert_gate_close, assert_keys_close, assert_mla_close, assert_scores_close,
                         dev_bits, score_magnitude,
                         device_status_clean, end_to_end, host_bits, mla_value_bound, run_step,
                         stagewise, workload)
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


# ----------------------------------------------------------------------------- configurations
@pytest.mark.parametrize("name", ["tiny", "batched"])
def test_config_stagewise_and_e2e(B, name):
    wl = workload(name)
    step, g = run_step(wl)
    rep = stagewise(wl, g)
    e2e = end_to_end(wl, g)
    print(name, rep, e2e)
    device_status_clean(B)


def test_config_ragged(B):
    wl = workload("ragged")
    step, g = run_step(wl)
    rep = stagewise(wl, g)
    print("ragged", rep, end_to_end(wl, g))
    device_status_clean(B)


def test_config_long_context(B):
    wl = workload("long")
    step, g = run_step(wl)
    rep = stagewise(wl, g)
    print("long", rep, end_to_end(wl, g))
    device_status_clean(B)


def test_config_prefill(B):
    """2048 queries: gate, scores, top-k and expand for every query; the end-to-end
    check compares the MLA output of every query whose selection agrees with the
    oracle's; the stage-wise MLA check on the GPU's own ids takes a sample."""
    wl = workload("prefill")
    step, g = run_step(wl)
    sample = np.r_[0:8, 1020:1028, 2040:2048]
    assert_gate_close(g["gate_w"], O.head_gate(wl.hidden, wl.w_gate))
    rep = stagewise(wl, g, queries=sample)
    # top-k + expand for every query (bit-exact)
    top, ids = O.topk_expand(g["scores"], g["cand"], g["pool_idx"], wl.q_req, wl.select_k)
    np.testing.assert_array_equal(g["top_pools"], top)
    np.testing.assert_array_equal(g["token_ids"], ids)
    # causality: every selected token is at or before its query's position
    sel = g["token_ids"]
    assert ((sel < 0) | (sel <= wl.q_pos[:, None])).all()
    e2e = end_to_end(wl, g)
    assert e2e["agree"] > 0
    print("prefill", rep, e2e)
    device_status_clean(B)


# ----------------------------------------------------------------------------- edge cases
def _mini(kpool, lengths, pads, holes=None, select_k=8, hm=16, seed=3, max_pools=None):
    lengths = list(lengths)
    if max_pools is None:
        max_pools = max(1, max((t + kpool - 1) // kpool for t in lengths))
    qr = list(range(len(lengths)))
    qp = [max(t - 1, 0) for t in lengths]
    return W.build(f"edge k{kpool}", lengths=lengths, pads=pads, kpool=kpool, max_pools=max_pools,
                   select_k=select_k, hm=hm, q_req=qr, q_pos=qp, seed=seed, holes=holes)


@pytest.mark.parametrize("kpool", [1, 2, 3, 4, 5, 6, 7, 8])
def test_every_kpool_with_ragged_requests(B, kpool):
    lengths = [1, kpool - 1 if kpool > 1 else 2, 37, 300, 129, 0, 520]
    pads = [0, 0, 5, 17, 129, 0, 3]          # request 4 is entirely padding; 5 is empty
    wl = _mini(kpool, lengths, pads, holes=[1 + 37 + 40, 1 + 37 + 41], select_k=16)
    step, g = run_step(wl)
    stagewise(wl, g)
    assert g["first_valid"][4] == 129 and g["first_valid"][5] == 0
    assert (g["top_pools"][4] == -1).all() and (g["token_ids"][5] == -1).all()
    device_status_clean(B)


@pytest.mark.parametrize("kpool,n_req,max_len,max_pools",
                         [(4, 2100, 60, 16), (8, 1200, 60, 16), (3, 300, 60, 16),
                          (4, 300, 2000, 512), (8, 90, 3000, 400)])
def test_compress_partitions(B, kpool, n_req, max_len, max_pools):
    """Request counts past the balanced partition's limit (2048 requests at kpool <= 4,
    1152 above) take the per-request tile grid, and so do requests whose pool counts
    lie within a tile of one another (lengths 0-60); lengths spread over hundreds of
    pools below the limit split the tiles holding pools evenly. Random padding, so
    many requests end in a partial pool, have no valid token or are empty."""
    rng = np.random.default_rng(n_req)
    lengths = rng.integers(0, max_len + 1, n_req).tolist()
    pads = [int(rng.integers(0, min(t, 100) + 1)) if t else 0 for t in lengths]
    wl = _mini(kpool, lengths, pads, select_k=4, max_pools=max_pools)
    step, g = run_step(wl)
    keys, idx, pv, fv = O.kpool_compress(wl.k, wl.gate, wl.valid, wl.req_start, wl.kpool,
                                         wl.max_pools, wl.ape, wl.ln_w, wl.ln_b, wl.eps)
    np.testing.assert_array_equal(g["first_valid"], fv)
    np.testing.assert_array_equal(g["pool_valid"], pv)
    np.testing.assert_array_equal(g["pool_idx"], idx)
    assert_keys_close(g["pool_keys"], keys, pv, wl, fv)
    device_status_clean(B)


def test_compress_gate_logits_far_apart(B):
    """Compress shifts each channel's softmax by slot 0's logit; where the slots'
    logits lie more than 2^7 apart (log2 units) a weight overflows and the warp
    redoes its pools shifted by the maximum. Gate logits of +-100 on some tokens
    (and 0.5 elsewhere) take that path; the keys still match the oracle."""
    for kpool in (4, 8):
        wl = _mini(kpool, [640, 333], [0, 5], select_k=8)
        g16 = wl.gate.copy()
        hi, lo = np.uint16(0x42C8), np.uint16(0xC2C8)        # bf16 +100, -100
        g16[3::7, ::3] = hi
        g16[5::11, 1::3] = lo
        wl.gate[:] = g16
        step, g = run_step(wl)
        keys, idx, pv, fv = O.kpool_compress(wl.k, wl.gate, wl.valid, wl.req_start, wl.kpool,
                                             wl.max_pools, wl.ape, wl.ln_w, wl.ln_b, wl.eps)
        np.testing.assert_array_equal(g["pool_valid"], pv)
        np.testing.assert_array_equal(g["pool_idx"], idx)
        assert_keys_close(g["pool_keys"], keys, pv, wl, fv)
    device_status_clean(B)


def test_select_more_than_candidates_and_sentinel(B):
    wl = _mini(4, [64, 40], [0, 10], select_k=64)
    step, g = run_step(wl)
    stagewise(wl, g)
    n0 = (g["top_pools"][0] >= 0).sum()
    assert n0 == 16 and (g["top_pools"][0][16:] == -1).all()
    assert (g["token_ids"][0][16 * 4:] == -1).all()
    device_status_clean(B)


def test_ties_break_to_lowest_pool_id(B):
    wl = _mini(4, [800], [0], select_k=32)
    wl.hidden[:] = 0.0          # gate weights 0 -> every candidate scores exactly 0
    step, g = run_step(wl)
    assert (g["gate_w"] == 0).all()
    stagewise(wl, g)
    assert list(g["top_pools"][0]) == list(range(32))
    device_status_clean(B)


@pytest.mark.parametrize("H", [16, 13])
def test_scores_many_queries(B, H):
    """300 queries (the many-query scores kernel at H = 16: groups of 16 queries
    sharing key tiles; the one-query kernel at H = 13): runs of one request that
    do not line up with the groups, queries naming no request, causal positions
    from before the first pool to past the last, 1000 pools (a ragged last tile).
    Every score and candidate flag against the oracle."""
    rng = np.random.default_rng(31 + H)
    Q, P, kp, Bn = 300, 1000, 4, 3
    q_req = np.sort(rng.integers(0, Bn, Q)).astype(np.int32)
    q_req[[5, 17, 200]] = [-1, 7, -3]
    fv = np.array([0, 3, 11], np.int32)
    q_pos = rng.integers(-5, P * kp + 20, Q).astype(np.int32)
    q_idx = W.f32_to_bf16_bits(rng.standard_normal((Q, H, 128)).astype(np.float32))
    keys = W.f32_to_bf16_bits(rng.standard_normal((Bn, P, 128)).astype(np.float32))
    pv = (rng.random((Bn, P)) < 0.9).astype(np.uint8)
    gw = rng.standard_normal((Q, H)).astype(np.float32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    scores = torch.full((Q, P), float("nan"), device="cuda")
    cand = torch.full((Q, P), 0x7F, dtype=torch.uint8, device="cuda")
    B.dsa_index_scores(dev_bits(q_idx), d(gw), d(q_req), d(q_pos), Q, H, 128, dev_bits(keys), d(pv),
                       d(fv), Bn, kp, P, scores, cand)
    torch.cuda.synchronize()
    ok = (q_req >= 0) & (q_req < Bn)
    gs, gc = scores.cpu().numpy(), cand.cpu().numpy()
    assert (gc[~ok] == 0).all() and np.isneginf(gs[~ok]).all()      # no request: no candidates
    sc, cd = O.index_scores(q_idx[ok], gw[ok], q_req[ok], q_pos[ok], keys, pv, fv, kp)
    np.testing.assert_array_equal(gc[ok], cd)
    assert_scores_close(gs[ok], sc, cd, score_magnitude(q_idx[ok], gw[ok], keys, q_req[ok]))
    device_status_clean(B)


def test_head_gate_shapes(B):
    rng = np.random.default_rng(5)
    # up to 592 rows the K split over clusters of 8; above, a CTA a 16-row block
    # over the whole of K (partial row blocks, K not a multiple of the 512-k
    # slice, N below 16)
    for M, K, N in [(1, 4096, 16), (5, 4096, 16), (16, 4096, 16), (17, 4096, 16),
                    (33, 1000, 8), (3, 4, 1), (2048, 4096, 16), (7, 8192, 13),
                    (600, 4100, 16), (1000, 1000, 13), (2047, 516, 16)]:
        h = rng.standard_normal((M, K), dtype=np.float32)
        w = (rng.standard_normal((K, N)) / 64).astype(np.float32)
        out = torch.full((M, N), float("nan"), device="cuda")
        B.dsa_head_gate(torch.from_numpy(h).cuda(), torch.from_numpy(w).cuda(), out, M, K, N)
        assert_gate_close(out.cpu().numpy(), O.head_gate(h, w), f"gate {M}x{K}x{N}")
    device_status_clean(B)


def test_topk_special_values_and_global_key_path(B):
    """Crafted scores: -0 vs +0 ties, NaN (ranks as -inf), -inf candidates, and a
    pool count above the shared-memory key cache (keys re-read from global)."""
    rng = np.random.default_rng(9)
    for P, K in [(300, 64), (40000, 512)]:
        Q = 3
        s = np.round(rng.standard_normal((Q, P)) * 2).astype(np.float32)
        s[0, ::7] = -0.0
        s[0, 1::7] = 0.0
        s[1, ::11] = np.nan
        s[1, 5::13] = -np.inf
        cand = (rng.random((Q, P)) < 0.9).astype(np.uint8)
        kp = 3
        pidx = (np.arange(P * kp, dtype=np.int32).reshape(1, P, kp) + 1)
        ref_top, ref_ids = O.topk_expand(s, cand, pidx, np.zeros(Q, np.int32), K)
        d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
        top = torch.empty(Q, K, dtype=torch.int32, device="cuda")
        ids = torch.empty(Q, K * kp, dtype=torch.int32, device="cuda")
        B.dsa_topk_expand(d(s), d(cand), d(pidx), d(np.zeros(Q, np.int32)), Q, 1, P, kp, K, top, ids)
        np.testing.assert_array_equal(top.cpu().numpy(), ref_top)
        np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    device_status_clean(B)


@pytest.mark.parametrize("hm", [16, 32, 48, 64, 128])
def test_mla_heads_and_id_edge_cases(B, hm):
    rng = np.random.default_rng(hm)
    lengths = [300, 90, 0]
    T = sum(lengths)
    rs = np.array([0, 300, 390, 390], np.int32)
    Wd = 200
    q = W.f32_to_bf16_bits(rng.standard_normal((4, hm, 512)).astype(np.float32))
    kv = W.f32_to_bf16_bits(rng.standard_normal((T, 512)).astype(np.float32))
    q_req = np.array([0, 1, 2, 0], np.int32)
    ids = np.full((4, Wd), -1, np.int32)
    ids[0, :150] = rng.choice(300, 150, replace=False)
    ids[0, 3] = 300                       # outside the request: ignored
    ids[1, :180:2] = rng.choice(90, 90, replace=False)
    ids[3, 7] = 123                       # one token
    scale = float(1 / np.sqrt(512))
    ref_out, ref_lse = O.sparse_mla(q, kv, rs, q_req, ids, scale)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = torch.empty(4, hm, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(4, hm, dtype=torch.float32, device="cuda")
    ws_n = B.dsa_sparse_mla_workspace_size(4, hm, Wd)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    B.dsa_sparse_mla_decode(dev_bits(q), dev_bits(kv), kv.shape[0], d(rs), d(q_req), d(ids), 4, 3,
                            hm, Wd, 512, 0, scale, out, lse, ws, ws_n)
    go, gl = host_bits(out), lse.cpu().numpy()
    assert_mla_close(go, ref_out, gl, ref_lse, vbound=mla_value_bound(kv, rs, q_req, ids))
    assert (go[2] == 0).all() and np.isneginf(gl[2]).all()      # empty request
    np.testing.assert_array_equal(go[3, 0], kv[123])                # single token: its row
    device_status_clean(B)


def test_mla_rows_past_kv_rows_are_not_read(B):
    # kv_rows bounds the cache: an id whose row falls at or past it counts as
    # invalid (it is neither read nor weighted). Request 1 owns rows 300..389;
    # the cache is declared to hold 350 rows, so its ids 50..89 drop out.
    rng = np.random.default_rng(11)
    hm, Wd = 64, 160
    rs = np.array([0, 300, 390], np.int32)
    kv_full = W.f32_to_bf16_bits(rng.standard_normal((390, 512)).astype(np.float32))
    q = W.f32_to_bf16_bits(rng.standard_normal((2, hm, 512)).astype(np.float32))
    q_req = np.array([0, 1], np.int32)
    ids = np.full((2, Wd), -1, np.int32)
    ids[0, :140] = rng.choice(300, 140, replace=False)
    ids[1, :90] = rng.permutation(90)
    kv_rows = 350
    ids_ref = ids.copy()
    ids_ref[1][(ids_ref[1] >= 0) & (rs[1] + ids_ref[1] >= kv_rows)] = -1
    scale = float(1 / np.sqrt(512))
    ref_out, ref_lse = O.sparse_mla(q, kv_full, rs, q_req, ids_ref, scale)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    out = torch.empty(2, hm, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(2, hm, dtype=torch.float32, device="cuda")
    ws_n = B.dsa_sparse_mla_workspace_size(2, hm, Wd)
    ws = torch.empty(max(ws_n, 16), dtype=torch.uint8, device="cuda")
    # the rows past kv_rows hold NaN on the device: reading any of them would show
    kv_dev = kv_full.copy()
    kv_dev[kv_rows:] = 0x7FC0
    B.dsa_sparse_mla_decode(dev_bits(q), dev_bits(kv_dev), kv_rows, d(rs), d(q_req), d(ids), 2, 2,
                            hm, Wd, 512, 0, scale, out, lse, ws, ws_n)
    assert np.isfinite(lse.cpu().numpy()).all()
    assert_mla_close(host_bits(out), ref_out, lse.cpu().numpy(), ref_lse,
                     vbound=mla_value_bound(kv_full, rs, q_req, ids_ref))
    device_status_clean(B)


def test_mla_launch_count(B):
    # one split: the split kernel alone; more: the combine kernel too
    assert B.dsa_sparse_mla_launch_count(148, 64, 2048) == 1
    assert B.dsa_sparse_mla_launch_count(2048, 64, 2048) == 1
    assert B.dsa_sparse_mla_launch_count(2, 64, 32768) == 2
    assert B.dsa_sparse_mla_launch_count(2, 64, 2048) == 2
    assert B.dsa_sparse_mla_launch_count(16, 64, 2048) == 2
    assert B.dsa_sparse_mla_launch_count(1, 16, 64) == 2        # two chunks, a split each
    assert B.dsa_sparse_mla_launch_count(0, 64, 2048) == 0


def test_maximum_select_k_and_kpool(B):
    """select_k = 4096 (the largest), kpool = 8: a 32768-id row, whose MLA splits 69 ways
    per query (138 CTAs) and merges more than 16 splits in the combine (its
    multi-round path)."""
    T = 40000
    wl = W.build("max select", lengths=[T, 700], pads=[3, 0], kpool=8, max_pools=(T + 7) // 8,
                 select_k=4096, hm=16, q_req=[0, 1], q_pos=[T - 1, 699], seed=23)
    assert wl.out_width == 32768
    assert B.dsa_sparse_mla_launch_count(2, 16, 32768) == 2
    step, g = run_step(wl)
    stagewise(wl, g)
    n0 = int((g["top_pools"][0] >= 0).sum())
    assert n0 == 4096                                    # 4999 candidate pools, 4096 taken
    assert int((g["top_pools"][1] >= 0).sum()) == 87     # request 1: all its 87 pools
    assert (g["token_ids"][1][87 * 8:] == -1).all()
    device_status_clean(B)
