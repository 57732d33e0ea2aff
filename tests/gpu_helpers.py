"""Shared helpers of the GPU parity tests: tolerances and device plumbing.

Tolerances (each derived from the arithmetic, see the docstrings):
  * fp32 head gate: |gpu - ref| <= 1e-5 * max(1, |ref|).
  * fp32 scores:    |gpu - ref| <= 1e-5 * max(1, S) with S = sum_h |g_h| relu(d_h),
                    the magnitude of the summed terms; the count beyond
                    1e-5 * max(1, |ref|) is reported beside it (cancelling terms).
  * bf16 pooled keys: |gpu - ref| <= ulp(ref) + max_s ulp(kn_s), at most 0.1 %
                    of elements beyond 1 ulp(ref) (one-ulp k_norm flips).
  * end to end (oracle from raw inputs): every score within its own bound (the
                    gate and arithmetic tolerances plus the propagated pooled-key
                    difference); a pool may be swapped only when that bound
                    explains the swap (see end_to_end in test_gpu_parity.py).
  * bf16 MLA out:   max-abs 2e-2 and |gpu - ref| <= ulp(ref) + (2^-8 + 2^-12) max_j |v_j[c]|
                    (bf16 softmax weights in the tensor-core PV product, bf16
                    split partials); lse 1e-4.
"""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle as O
from sparse_attention_indexer_head_b200 import workloads as W


def bf16f(bits) -> np.ndarray:
    return W.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (2^-133 in the subnormal range)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(ax)                  # ax = m 2^e, m in [0.5, 1)
    e = np.maximum(e - 1, -126)
    return np.ldexp(1.0, e - 7)


def assert_gate_close(gpu, ref, what="gate"):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    tol = 1e-5 * np.maximum(1.0, np.abs(ref))
    bad = np.argwhere(err > tol)
    assert bad.size == 0, f"{what}: {len(bad)} outside 1e-5*max(1,|ref|); worst {err.max():.3g}"
    return float(err.max())


def score_magnitude(q_idx_bits, gate_w, keys_bits, q_req, kpool=None):
    """S[q,p] = sum_h |g_h| * relu(<q_h, key_p>) in fp64 (for the scores tolerance)."""
    q = bf16f(q_idx_bits)                                   # [Q,H,D]
    keys = bf16f(keys_bits)                                 # [B,P,D]
    out = np.empty((q.shape[0], keys.shape[1]))
    for i in range(q.shape[0]):
        d = np.einsum("hc,pc->hp", q[i], keys[q_req[i]])
        out[i] = (np.abs(gate_w[i]).astype(np.float64)[:, None] * np.maximum(d, 0)).sum(0)
    return out


def assert_scores_close(gpu, ref, cand, mag):
    """Scores of candidates within 1e-5 * max(1, S), S = sum_h |g_h| relu(d_h) the
    magnitude of the summed terms; -inf exactly at non-candidates.

    The specification's 1e-5 * max(1, |ref|) is reported beside it (over_plain):
    an fp32 sum of terms of size S carries rounding of order 1e-7 * S whatever
    the order of the sum, so where the head terms cancel (|ref| far below S) it
    can exceed 1e-5 * |ref|. It does for a handful of scores among millions;
    the count and the worst ratio to that bound are returned.
    """
    cand = cand.astype(bool)
    assert np.isneginf(gpu[~cand]).all(), "scores of non-candidates must be -inf"
    g, r, m = gpu[cand].astype(np.float64), ref[cand].astype(np.float64), mag[cand]
    assert np.isfinite(g).all()
    err = np.abs(g - r)
    tol = 1e-5 * np.maximum(1.0, m)
    assert (err <= tol).all(), f"scores: {(err > tol).sum()} outside tolerance; worst {err.max():.3g}"
    plain = 1e-5 * np.maximum(1.0, np.abs(r))
    over = err > plain
    return dict(max_abs=float(err.max(initial=0)), n=int(cand.sum()), over_plain=int(over.sum()),
                worst_over_plain=float((err / plain).max(initial=0)),
                min_cancellation_over_plain=float((m[over] / np.maximum(1.0, np.abs(r[over]))).min(initial=np.inf)))


def kn_ulp_bound(k_bits, ln_w_bits, ln_b_bits, eps, rows):
    """max over a pool's slots of ulp_bf16(kn) per channel; rows: [n_pools, kpool] token rows."""
    x = bf16f(k_bits[rows.reshape(-1)])                     # [n*kp, D]
    mu = x.mean(-1, keepdims=True)
    var = ((x - mu) ** 2).mean(-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + np.float32(eps)) * bf16f(ln_w_bits) + bf16f(ln_b_bits)
    u = bf16_ulp(y * (1 + 2.0 ** -8))                      # a hair above: covers the rounded value
    return u.reshape(rows.shape[0], rows.shape[1], -1).max(1)


def assert_keys_close(gpu_keys, ref_keys, pool_valid, wl, first_valid):
    """Pooled keys of valid pools: |gpu - ref| <= ulp(ref) + max_s ulp(kn_s), and at
    most 0.1 % of the elements more than 1 ulp(ref) away.

    The kernel takes each token's LayerNorm mean and rstd in fp32 and rounds
    kn = (k - mu) * rstd * w + b to bf16 as the specification stores it. Where the exact kn
    lies within fp32 error of a bf16 rounding boundary, the two roundings can
    differ by one bf16 ulp of kn; that kn enters the pooled value with its
    softmax weight w_s <= 1, moving it by at most w_s * ulp(kn_s) <= max_s
    ulp(kn_s) before the final rounding, which adds at most ulp(ref). A flip
    needs the exact kn within fp32 error (about 2^-21 relative) of a bf16
    boundary, about one kn in 2^12, and it carries a pooled element more than
    1 ulp(ref) away only when that element also lies near its own boundary:
    the 0.1 % cap on such elements is far above what that allows.
    """
    b_idx, p_idx = np.nonzero(pool_valid)
    if b_idx.size == 0:
        return dict(n=0)
    g = bf16f(gpu_keys[b_idx, p_idx])
    r = bf16f(ref_keys[b_idx, p_idx])
    rs = wl.req_start[b_idx].astype(np.int64) + first_valid[b_idx] + p_idx.astype(np.int64) * wl.kpool
    rows = rs[:, None] + np.arange(wl.kpool)[None, :]
    bound = bf16_ulp(r) + kn_ulp_bound(wl.k, wl.ln_w, wl.ln_b, wl.eps, rows)
    err = np.abs(g - r)
    assert (err <= bound).all(), f"pool keys: {(err > bound).sum()} outside ulp bound"
    over1 = int((err > bf16_ulp(r)).sum())
    frac = over1 / err.size
    assert frac < 1e-3, f"pool keys: {over1} of {err.size} elements beyond 1 ulp"
    return dict(n=int(err.size), exact=float((err == 0).mean()), over_1ulp=over1)


def mla_value_bound(kv_bits, req_start, q_req, token_ids):
    """max_j |v_j[c]| over each query's selected latent rows: [Q, 512] (0 if none)."""
    kv = bf16f(kv_bits) if kv_bits.dtype == np.uint16 else kv_bits
    out = np.zeros((len(q_req), kv.shape[1]))
    for i, b in enumerate(q_req):
        T = req_start[b + 1] - req_start[b]
        ids = token_ids[i][(token_ids[i] >= 0) & (token_ids[i] < T)]
        if ids.size:
            out[i] = np.abs(kv[req_start[b] + ids]).max(0)
    return out


def assert_mla_close(gpu_out, ref_out, gpu_lse, ref_lse, vbound=None, rows=None):
    """MLA output parity.

    The tensor-core PV product takes the softmax weights as bf16, so each weight
    carries a relative rounding error of at most 2^-9. With the row sum taken
    from the unrounded weights, out' - out = sum_j w_j e_j v_j / sum_j w_j, so
    |out' - out| <= 2^-9 max_j |v_j[c]|. When a query's splits merge through
    the workspace, each split's O row is stored as bf16 once more: another
    relative 2^-9 of |O_s[c]| <= l_s max_j |v_j[c]|, i.e. at most
    2^-9 max_j |v_j[c]| after the merge. The bound used is ulp(ref) plus
    (2^-8 + 2^-12) max_j |v_j[c]|: the two roundings and a margin for fp32
    accumulation and the exp2 approximation, which are far below 2^-12.
    Also the stated max-abs 2e-2, and lse within 1e-4 (fp32 sums of
    fp32 weights; one missing token among 2048 moves lse by ~1e-3).
    """
    g, r = bf16f(gpu_out), bf16f(ref_out)
    if rows is not None:
        g, r = g[rows], r[rows]
        gpu_lse, ref_lse = gpu_lse[rows], ref_lse[rows]
        if vbound is not None:
            vbound = vbound[rows]
    err = np.abs(g - r)
    assert err.max(initial=0) <= 2e-2, f"mla out max-abs {err.max():.3g}"
    if vbound is not None:
        bound = bf16_ulp(r) + (2.0 ** -8 + 2.0 ** -12) * vbound[:, None, :]
        assert (err <= bound).all(), f"mla out: {(err > bound).sum()} outside the weight-rounding bound"
    within = float((err <= bf16_ulp(r)).mean()) if err.size else 1.0
    both_inf = np.isneginf(gpu_lse) & np.isneginf(ref_lse)
    assert (np.isneginf(gpu_lse) == np.isneginf(ref_lse)).all()
    lerr = np.abs(gpu_lse[~both_inf] - ref_lse[~both_inf])
    assert lerr.max(initial=0) <= 1e-4, f"lse max-abs {lerr.max():.3g}"
    return dict(max_abs=float(err.max(initial=0)), rms=float(np.sqrt((err ** 2).mean())) if err.size else 0.0,
                within_1ulp=within, lse_max=float(lerr.max(initial=0)))


@functools.lru_cache(maxsize=8)
def workload(name: str, **kw):
    return W.make(name, **kw)


def device_status_clean(B):
    assert B.dsa_device_status(reset=True) == 0, "a kernel gave up a bounded wait"


def dev_bits(x: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit array -> device bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


# ----------------------------------------------------------------------------- path checks
def run_step(wl, canary=True, fused=False):
    """One step of the path on the workload (the fused indexer when fused is set),
    with every output first filled with 0x7F bytes so a missed write shows."""
    from sparse_attention_indexer_head_b200.pipeline import DecodeStep
    step = DecodeStep(wl, fused_indexer=fused)
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
    within 1e-5 max(1, S) of its exact value (the stage-wise tolerance, S the
    size of its summed terms),
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
        S = np.abs(gg[i]) @ dg                                 # size of the GPU's summed terms
        out[i] = (1e-5 * np.maximum(1.0, S) + np.abs(gg[i] - gr[i]) @ dg
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
    size of the score's terms), so swaps stay within the specification's score
    gap. Rows
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
    err = np.zeros_like(sr)
    err[cand] = np.abs(s_gpu[cand] - sr[cand])
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
