"""The fused indexer (dsa_indexer_select: head gate, scores, top-k and expansion
in one launch of one thread-block cluster per query) against the CPU oracle.

Stage by stage, as for the separate calls: the gate against orc_head_gate; the
scores and candidate flags against orc_index_scores fed the kernel's own gate
and pooled keys; the selection and token ids, bit-exact, against
orc_topk_expand fed the kernel's own scores. Every output starts filled with
0x7F bytes, so an element the kernel fails to write shows.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_helpers import (assert_gate_close, assert_scores_close, device_status_clean, end_to_end,
                         run_step, score_magnitude, stagewise, workload)
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


@pytest.mark.parametrize("name", ["tiny", "batched", "ragged", "long"])
def test_fused_step_decode_configs(B, name):
    wl = workload(name)
    step, g = run_step(wl, fused=True)
    assert step.kernels_per_step() == 1 + 1 + B.dsa_sparse_mla_launch_count(wl.Q, wl.hm, wl.out_width)
    rep = stagewise(wl, g)
    print(name, rep, end_to_end(wl, g))
    device_status_clean(B)


def test_fused_step_prefill(B):
    """2048 queries of one request: gate, scores, top-k and expansion for every query
    (the stage-wise MLA check on a sample)."""
    wl = workload("prefill")
    step, g = run_step(wl, fused=True)
    assert_gate_close(g["gate_w"], O.head_gate(wl.hidden, wl.w_gate))
    sc, cd = O.index_scores(wl.q_idx, g["gate_w"], wl.q_req, wl.q_pos, g["pool_keys"],
                            g["pool_valid"], g["first_valid"], wl.kpool)
    np.testing.assert_array_equal(g["cand"], cd)
    assert_scores_close(g["scores"], sc, cd,
                        score_magnitude(wl.q_idx, g["gate_w"], g["pool_keys"], wl.q_req))
    top, ids = O.topk_expand(g["scores"], g["cand"], g["pool_idx"], wl.q_req, wl.select_k)
    np.testing.assert_array_equal(g["top_pools"], top)
    np.testing.assert_array_equal(g["token_ids"], ids)
    stagewise(wl, g, queries=np.r_[0:4, 1022:1026, 2044:2048])
    device_status_clean(B)


def _mini(kpool, lengths, pads, select_k, max_pools=None, holes=None, seed=5, q_req=None,
          q_pos=None):
    lengths = list(lengths)
    if max_pools is None:
        max_pools = max(1, max((t + kpool - 1) // kpool for t in lengths))
    qr = list(range(len(lengths))) if q_req is None else list(q_req)
    qp = [max(lengths[b] - 1, 0) if 0 <= b < len(lengths) else 0 for b in qr] if q_pos is None \
        else list(q_pos)
    return W.build(f"indexer edge k{kpool}", lengths=lengths, pads=pads, kpool=kpool,
                   max_pools=max_pools, select_k=select_k, hm=16, q_req=qr, q_pos=qp, seed=seed,
                   holes=holes)


@pytest.mark.parametrize("kpool", [1, 3, 4, 8])
def test_cluster_sizes_and_ragged_requests(B, kpool):
    # 4201 pool slots: 33 tiles of 128, so a cluster of 8 CTAs with 5 tiles each
    # but the last two (3 tiles, none); requests from a few pools to 4200, one all
    # padding and one empty
    lengths = [37, 300 * kpool, 129, 0, 4200 * kpool + 3]
    pads = [5, 17, 129, 0, 3]
    wl = _mini(kpool, lengths, pads, select_k=300, holes=[37 + 40, 37 + 41])
    step, g = run_step(wl, fused=True)
    stagewise(wl, g)
    assert g["first_valid"][2] == 129
    assert (g["top_pools"][2] == -1).all() and (g["token_ids"][3] == -1).all()
    device_status_clean(B)


@pytest.mark.parametrize("kpool,lengths,pads,select_k", [
    # 300 pool slots: 3 tiles, so five of the cluster's eight CTAs hold no pool
    # and send empty counts; one request shorter than select_k, one all padding,
    # one empty
    (4, [37, 1200, 129, 0, 1100], [5, 17, 129, 0, 2], 100),
    # 2048 pool slots (the batched decode's count): two tiles a CTA
    (1, [2048, 700, 5], [0, 3, 5], 512),
    (8, [16384, 9000], [7, 0], 512),
])
def test_small_pool_counts_and_idle_ranks(B, kpool, lengths, pads, select_k):
    wl = _mini(kpool, lengths, pads, select_k=select_k, holes=[37 + 40, 37 + 41, 400])
    assert wl.max_pools <= 2048
    step, g = run_step(wl, fused=True)
    stagewise(wl, g)
    device_status_clean(B)


def test_ties_and_more_slots_than_candidates(B):
    # a zero gate scores every candidate exactly 0: the lowest pool ids win, and a
    # request with fewer candidates than select_k gets the -1 tail
    wl = _mini(4, [3000, 90], [0, 6], select_k=64)
    wl.hidden[:] = 0.0
    step, g = run_step(wl, fused=True)
    assert (g["gate_w"] == 0).all()
    stagewise(wl, g)
    assert list(g["top_pools"][0]) == list(range(64))
    n1 = int((g["top_pools"][1] >= 0).sum())
    assert n1 == (90 - 6) // 4 and (g["token_ids"][1][n1 * 4:] == -1).all()
    device_status_clean(B)


def test_out_of_range_request_and_causal_positions(B):
    # query 1 names no request (no candidates, every slot -1); queries 2-4 sit at
    # earlier positions of request 0 (causal candidate boundary)
    wl = _mini(4, [2000, 500], [0, 0], select_k=100, q_req=[0, 7, 0, 0, 0],
               q_pos=[1999, 0, 3, 400, 401])
    step, g = run_step(wl, fused=True)
    assert (g["cand"][1] == 0).all() and np.isneginf(g["scores"][1]).all()
    assert (g["top_pools"][1] == -1).all() and (g["token_ids"][1] == -1).all()
    assert g["cand"][2].sum() == 1                       # only pool 0 ends by position 3
    qs = [0, 2, 3, 4]
    ref_gate = O.head_gate(wl.hidden, wl.w_gate)
    assert_gate_close(g["gate_w"], ref_gate)
    sc, cd = O.index_scores(wl.q_idx[qs], g["gate_w"][qs], wl.q_req[qs], wl.q_pos[qs],
                            g["pool_keys"], g["pool_valid"], g["first_valid"], wl.kpool)
    np.testing.assert_array_equal(g["cand"][qs], cd)
    assert_scores_close(g["scores"][qs], sc, cd,
                        score_magnitude(wl.q_idx[qs], g["gate_w"][qs], g["pool_keys"], wl.q_req[qs]))
    top, ids = O.topk_expand(g["scores"][qs], g["cand"][qs], g["pool_idx"], wl.q_req[qs], wl.select_k)
    np.testing.assert_array_equal(g["top_pools"][qs], top)
    np.testing.assert_array_equal(g["token_ids"][qs], ids)
    device_status_clean(B)


def test_direct_call_odd_gate_shape(B):
    """Through the binding with H = 7 heads and K = 1000 (the gate's scalar path)."""
    rng = np.random.default_rng(3)
    Q, H, K, kp, P, SK = 3, 7, 1000, 2, 700, 50
    Bn = 2
    hidden = rng.standard_normal((Q, K), dtype=np.float32)
    w = (rng.standard_normal((K, H)) / 32).astype(np.float32)
    q_idx = W.f32_to_bf16_bits(rng.standard_normal((Q, H, 128)).astype(np.float32))
    keys = W.f32_to_bf16_bits(rng.standard_normal((Bn, P, 128)).astype(np.float32))
    pv = (rng.random((Bn, P)) < 0.9).astype(np.uint8)
    fv = np.array([0, 11], np.int32)
    pidx = (np.arange(Bn * P * kp, dtype=np.int32).reshape(Bn, P, kp) % 5000)
    q_req = np.array([0, 1, 1], np.int32)
    q_pos = np.array([2 * P - 1, 2 * P + 10, 900], np.int32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    gate_w = torch.full((Q, H), float("nan"), device="cuda")
    scores = torch.full((Q, P), float("nan"), device="cuda")
    cand = torch.full((Q, P), 0x7F, dtype=torch.uint8, device="cuda")
    top = torch.full((Q, SK), 0x7F7F7F7F, dtype=torch.int32, device="cuda")
    ids = torch.full((Q, SK * kp), 0x7F7F7F7F, dtype=torch.int32, device="cuda")
    B.dsa_indexer_select(d(hidden), d(w), K, bits(q_idx), d(q_req), d(q_pos), Q, H, 128, bits(keys),
                         d(pv), d(fv), d(pidx), Bn, kp, P, SK, gate_w, scores, cand, top, ids)
    torch.cuda.synchronize()
    gw = gate_w.cpu().numpy()
    assert_gate_close(gw, O.head_gate(hidden, w))
    sc, cd = O.index_scores(q_idx, gw, q_req, q_pos, keys, pv, fv, kp)
    np.testing.assert_array_equal(cand.cpu().numpy(), cd)
    assert_scores_close(scores.cpu().numpy(), sc, cd, score_magnitude(q_idx, gw, keys, q_req))
    rt, ri = O.topk_expand(scores.cpu().numpy(), cand.cpu().numpy(), pidx, q_req, SK)
    np.testing.assert_array_equal(top.cpu().numpy(), rt)
    np.testing.assert_array_equal(ids.cpu().numpy(), ri)
    device_status_clean(B)


@pytest.mark.parametrize("Q", [4, 10])
def test_direct_call_largest_pool_count(B, Q):
    """32768 pools a request (the largest the fused call takes): 4 queries run as
    clusters of 16 CTAs with a deep key ring, 10 as clusters of 8 whose ring the
    shared-memory limit bounds; every output against the oracle stages."""
    rng = np.random.default_rng(Q)
    H, K, kp, P, SK, Bn = 16, 4096, 4, 32768, 512, Q
    hidden = rng.standard_normal((Q, K), dtype=np.float32)
    w = (rng.standard_normal((K, H)) / 64).astype(np.float32)
    q_idx = W.f32_to_bf16_bits(rng.standard_normal((Q, H, 128)).astype(np.float32))
    keys = W.f32_to_bf16_bits(rng.standard_normal((Bn, P, 128)).astype(np.float32))
    pv = (rng.random((Bn, P)) < 0.95).astype(np.uint8)
    fv = rng.integers(0, 4, Bn).astype(np.int32)
    pidx = (np.arange(Bn * P * kp, dtype=np.int64).reshape(Bn, P, kp) % (1 << 30)).astype(np.int32)
    q_req = np.arange(Q, dtype=np.int32)
    q_pos = (fv + kp * P - 1 - rng.integers(0, 5000, Q)).astype(np.int32)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bits = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    gate_w = torch.full((Q, H), float("nan"), device="cuda")
    scores = torch.full((Q, P), float("nan"), device="cuda")
    cand = torch.full((Q, P), 0x7F, dtype=torch.uint8, device="cuda")
    top = torch.full((Q, SK), 0x7F7F7F7F, dtype=torch.int32, device="cuda")
    ids = torch.full((Q, SK * kp), 0x7F7F7F7F, dtype=torch.int32, device="cuda")
    B.dsa_indexer_select(d(hidden), d(w), K, bits(q_idx), d(q_req), d(q_pos), Q, H, 128, bits(keys),
                         d(pv), d(fv), d(pidx), Bn, kp, P, SK, gate_w, scores, cand, top, ids)
    torch.cuda.synchronize()
    gw = gate_w.cpu().numpy()
    assert_gate_close(gw, O.head_gate(hidden, w))
    sc, cd = O.index_scores(q_idx, gw, q_req, q_pos, keys, pv, fv, kp)
    np.testing.assert_array_equal(cand.cpu().numpy(), cd)
    assert_scores_close(scores.cpu().numpy(), sc, cd, score_magnitude(q_idx, gw, keys, q_req))
    rt, ri = O.topk_expand(scores.cpu().numpy(), cand.cpu().numpy(), pidx, q_req, SK)
    np.testing.assert_array_equal(top.cpu().numpy(), rt)
    np.testing.assert_array_equal(ids.cpu().numpy(), ri)
    device_status_clean(B)
