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
from gpu_helpers import (assert_gate_close, assert_keys_close, assert_mla_close,
                         assert_scores_close, bf16f, dev_bits, device_status_clean, host_bits,
                         mla_value_bound, score_magnitude, workload)
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


def run_step(wl, canary=True):
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    step = DecodeStep(wl)
    if canary:   # every output the contract says is written must lose the 0x7F fill
        for t in (step.gate_w, step.pool_idx, step.pool_valid, step.first_valid, step.scores,
                  step.cand, step.top_pools, step.token_ids, step.out, step.lse):
            t.view(torch.uint8).fill_(0x7F)
    step.run()
    torch.cuda.synchronize()
    return step, step.outputs_numpy()


def stagewise(wl, g, queries=None):
    """Each oracle stage on the GPU's inputs to that stage; returns a report dict."""
    rep = {}
    qs = np.arange(wl.Q) if queries is None else np.asarray(queries)
    # a1
    ref_gate = O.head_gate(wl.hidden[qs], wl.w_gate)
    rep["gate_max_abs"] = assert_gate_close(g["gate_w"][qs], ref_gate)
    # a2+a3
    keys, idx, pv, fv = O.kpool_compress(wl.k, wl.gate, wl.valid, wl.req_start, wl.kpool,
                                         wl.max_pools, wl.ape, wl.ln_w, wl.ln_b, wl.eps)
    np.testing.assert_array_equal(g["first_valid"], fv)
    np.testing.assert_array_equal(g["pool_valid"], pv)
    np.testing.assert_array_equal(g["pool_idx"], idx)
    rep["keys"] = assert_keys_close(g["pool_keys"], keys, pv, wl, fv)
    # a4 on GPU gate_w and GPU pool tensors
    sc, cd = O.index_scores(wl.q_idx[qs], g["gate_w"][qs], wl.q_req[qs], wl.q_pos[qs],
                            g["pool_keys"], g["pool_valid"], g["first_valid"], wl.kpool)
    np.testing.assert_array_equal(g["cand"][qs], cd)
    mag = score_magnitude(wl.q_idx[qs], g["gate_w"][qs], g["pool_keys"], wl.q_req[qs])
    rep["scores"] = assert_scores_close(g["scores"][qs], sc, cd, mag)
    # a5+a6 on GPU scores: bit-exact
    top, ids = O.topk_expand(g["scores"][qs], g["cand"][qs], g["pool_idx"], wl.q_req[qs],
                             wl.select_k)
    np.testing.assert_array_equal(g["top_pools"][qs], top)
    np.testing.assert_array_equal(g["token_ids"][qs], ids)
    # a7 on GPU token ids
    out, lse = O.sparse_mla(wl.q_mla[qs], wl.kv, wl.req_start, wl.q_req[qs], g["token_ids"][qs],
                            wl.sm_scale)
    vb = mla_value_bound(wl.kv, wl.req_start, wl.q_req[qs], g["token_ids"][qs])
    rep["mla"] = assert_mla_close(g["out"][qs], out, g["lse"][qs], lse, vbound=vb)
    return rep


def e2e_score_bound(wl, qs, g, gate_ref, keys_ref):
    """Per-pool bound of |GPU score - oracle score from raw inputs|, [len(qs), P].

    The GPU scores a pool from its own head gate and pooled keys; the oracle
    from its own. In exact arithmetic the two scores differ by
      sum_h (g_gpu_h - g_ref_h) relu(d_gpu_h) + sum_h g_ref_h (relu(d_gpu_h) - relu(d_ref_h))
    (d: the head dots with each side's pooled key), and the GPU's fp32 score is
    within 1e-5 max(1, |score|) of its exact value (the stage-wise tolerance),
    the oracle's within half an fp32 ulp. The bound is the sum of those terms'
    magnitudes: where both sides hold the same pooled key it is the gate and
    arithmetic tolerances alone.
    """
    q = bf16f(wl.q_idx[qs])
    kg, kr = bf16f(g["pool_keys"]), bf16f(keys_ref)
    gg = g["gate_w"][qs].astype(np.float64)
    gr = gate_ref.astype(np.float64)
    out = np.zeros((len(qs), kg.shape[1]))
    for i in range(len(qs)):
        b = wl.q_req[qs[i]]
        dg = np.maximum(q[i] @ kg[b].T, 0.0)                 # [H, P]
        dr = np.maximum(q[i] @ kr[b].T, 0.0)
        s_exact = gg[i] @ dg
        out[i] = (1e-5 * np.maximum(1.0, np.abs(s_exact)) + np.abs(gg[i] - gr[i]) @ dg
                  + np.abs(gr[i]) @ np.abs(dg - dr) + 2.0 ** -24 * np.abs(gr[i] @ dr))
    return out


def end_to_end(wl, g, queries=None):
    """Oracle from raw inputs vs the GPU.

    Validity, candidates and pool indices are bit-exact. Every candidate's GPU
    score lies within its bound E (e2e_score_bound). The selections may differ
    only by swaps that those bounds explain: for every pool p the oracle selects
    and the GPU does not, and every pool p' the GPU selects and the oracle does
    not, s_ref[p] - E[p] <= s_ref[p'] + E[p']. Where both sides hold the same
    pooled keys, E is the gate and arithmetic tolerance (about 2e-5 of the
    score's terms), so swaps stay within the specification's score gap. Rows
    whose selections agree have bit-exact token ids and their MLA output is
    compared with the oracle's.
    """
    qs = np.arange(wl.Q) if queries is None else np.asarray(queries)
    gate_ref = O.head_gate(wl.hidden[qs], wl.w_gate)
    keys, idx, pv, fv = O.kpool_compress(wl.k, wl.gate, wl.valid, wl.req_start, wl.kpool,
                                         wl.max_pools, wl.ape, wl.ln_w, wl.ln_b, wl.eps)
    np.testing.assert_array_equal(g["pool_valid"], pv)
    np.testing.assert_array_equal(g["pool_idx"], idx)
    np.testing.assert_array_equal(g["first_valid"], fv)
    s_ref, c_ref = O.index_scores(wl.q_idx[qs], gate_ref, wl.q_req[qs], wl.q_pos[qs], keys, pv, fv,
                                  wl.kpool)
    np.testing.assert_array_equal(g["cand"][qs], c_ref)
    top_ref, ids_ref = O.topk_expand(s_ref, c_ref, idx, wl.q_req[qs], wl.select_k)
    E = e2e_score_bound(wl, qs, g, gate_ref, keys)
    cand = c_ref.astype(bool)
    s_gpu = g["scores"][qs].astype(np.float64)
    sr = s_ref.astype(np.float64)
    err = np.abs(s_gpu - sr)
    assert (err[cand] <= E[cand]).all(), f"{(err[cand] > E[cand]).sum()} scores outside their bound"
    agree_rows = []
    swaps = 0
    for i, q in enumerate(qs):
        a = set(top_ref[i][top_ref[i] >= 0].tolist())
        gs = set(g["top_pools"][q][g["top_pools"][q] >= 0].tolist())
        assert len(a) == len(gs)
        if a == gs:
            agree_rows.append(i)
            np.testing.assert_array_equal(g["token_ids"][q], ids_ref[i])
            continue
        out_, in_ = np.array(sorted(a - gs)), np.array(sorted(gs - a))
        swaps += len(out_)
        worst_out = (sr[i, out_] - E[i, out_]).max()
        best_in = (sr[i, in_] + E[i, in_]).min()
        assert worst_out <= best_in, (int(q), worst_out, best_in)
    if agree_rows:
        rows = np.asarray(agree_rows)
        out, lse = O.sparse_mla(wl.q_mla[qs[rows]], wl.kv, wl.req_start, wl.q_req[qs[rows]],
                                ids_ref[rows], wl.sm_scale)
        vb = mla_value_bound(wl.kv, wl.req_start, wl.q_req[qs[rows]], ids_ref[rows])
        assert_mla_close(g["out"][qs[rows]], out, g["lse"][qs[rows]], lse, vbound=vb)
    return dict(swaps=swaps, agree=len(agree_rows), max_err_over_bound=float((err[cand] / E[cand]).max()))


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


def test_head_gate_shapes(B):
    rng = np.random.default_rng(5)
    for M, K, N in [(1, 4096, 16), (5, 4096, 16), (16, 4096, 16), (17, 4096, 16),
                    (33, 1000, 8), (3, 4, 1), (2048, 4096, 16), (7, 8192, 13)]:
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
    # one split: the split kernel alone; more than 8 splits: always the workspace
    # merge, so a combine kernel too; 2..8 splits: 1 or 2 (clusters where they fit)
    assert B.dsa_sparse_mla_launch_count(148, 64, 2048) == 1
    assert B.dsa_sparse_mla_launch_count(2, 64, 2048) == 2
    assert B.dsa_sparse_mla_launch_count(16, 64, 2048) in (1, 2)
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
