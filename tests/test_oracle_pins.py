"""Pins of the CPU oracle to things other than itself (no GPU).

Each test ties one oracle stage to brute force, a closed form, a library
routine, or an invariant the pages state, chosen so that a plausible slip in
the oracle (a dropped term, a wrong axis, sign or index, a missing offset)
fails at least one of them. Page passages are cited by page title and section:
  "spark_model/layers/glm5next_dsa/mod.rs" (mod.rs) and
  "feat(glm53): indexer fp32 head-gate split-K" (PR #227).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from sparse_attention_indexer_head_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16_values(bits):
    return W.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def rnd_bf16(orc, x):
    x = np.asarray(x, dtype=np.float64)
    return np.array([orc.bf16_from_f64(v) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)


def bf16_nearest_even_bruteforce(x: float) -> int:
    """Nearest bf16 by exact rational distance; ties to the even bit pattern."""
    f32 = np.array([x], dtype=np.float32)
    if not np.isfinite(f32[0]):
        f32 = np.array([np.sign(x) * np.finfo(np.float32).max], dtype=np.float32)
    centre = int(f32.view(np.uint32)[0] >> 16)
    best = None
    fx = Fraction(x)
    for b in range(centre - 3, centre + 4):
        b &= 0xFFFF
        v = float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])
        if not math.isfinite(v):
            continue
        d = abs(Fraction(v) - fx)
        key = (d, b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return best[1]


# --------------------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_matches_bruteforce(orc):
    rng = np.random.default_rng(11)
    xs = list(rng.standard_normal(400) * np.exp(rng.uniform(-30, 30, 400)))
    # exact midpoints between neighbouring bf16 values (the tie cases)
    for b in rng.integers(0x0080, 0x7F00, 200):
        lo = bf16_values([b])[0]
        hi = bf16_values([b + 1])[0]
        xs.append((lo + hi) / 2)
        xs.append(-(lo + hi) / 2)
    # subnormal bf16 range and its ties
    for b in rng.integers(1, 0x7F, 50):
        lo, hi = bf16_values([b])[0], bf16_values([b + 1])[0]
        xs += [(lo + hi) / 2, lo * 1.3, hi * 0.7]
    for x in xs:
        assert orc.bf16_from_f64(x) == bf16_nearest_even_bruteforce(x), x


def test_bf16_rounding_specials(orc):
    mx = bf16_values([0x7F7F])[0]
    half_ulp = (bf16_values([0x7F7F])[0] - bf16_values([0x7F7E])[0]) / 2
    assert orc.bf16_from_f64(mx) == 0x7F7F
    assert orc.bf16_from_f64(mx + half_ulp * 0.999) == 0x7F7F
    assert orc.bf16_from_f64(mx + half_ulp) == 0x7F80          # tie goes to even -> inf
    assert orc.bf16_from_f64(-(mx + 2 * half_ulp)) == 0xFF80
    assert orc.bf16_from_f64(0.0) == 0 and orc.bf16_from_f64(-0.0) == 0x8000
    assert orc.bf16_from_f64(1.0) == 0x3F80
    assert orc.bf16_from_f64(1.0 + 2.0 ** -8) == 0x3F80          # tie -> even (down)
    assert orc.bf16_from_f64(1.0 + 3 * 2.0 ** -8) == 0x3F82      # tie -> even (up)
    assert orc.bf16_from_f64(2.0 ** -140) == 0                    # below half the min subnormal
    assert orc.f64_from_bf16(0x3F80) == 1.0


# --------------------------------------------------------------------------- a1 head gate
def test_head_gate_is_correctly_rounded_dot(orc):
    """PR #227: out = hidden @ W in fp32. Exact sums (math.fsum) rounded once to fp32."""
    rng = np.random.default_rng(1)
    M, K, N = 3, 4096, 16
    hidden = rng.standard_normal((M, K), dtype=np.float32)
    w = (rng.standard_normal((K, N), dtype=np.float32) / np.float32(64))
    out = orc.head_gate(hidden, w)
    prod = hidden.astype(np.float64)[:, :, None] * w.astype(np.float64)[None, :, :]
    for m in range(M):
        for n in range(N):
            exact = np.float32(math.fsum(prod[m, :, n]))
            assert abs(out[m, n] - exact) <= abs(np.spacing(exact)), (m, n)


def test_head_gate_vs_library_matmul(orc):
    rng = np.random.default_rng(2)
    hidden = rng.standard_normal((5, 96), dtype=np.float32)
    w = rng.standard_normal((96, 7), dtype=np.float32)
    ref = torch.from_numpy(hidden).double() @ torch.from_numpy(w).double()
    np.testing.assert_allclose(orc.head_gate(hidden, w), ref.float().numpy(), rtol=2e-7, atol=1e-7)
    # orientation: a one-hot row picks a row of W
    e = np.zeros((1, 96), np.float32)
    e[0, 17] = 1
    np.testing.assert_array_equal(orc.head_gate(e, w)[0], w[17])


# --------------------------------------------------------------------------- a2 k_norm
def _compress(orc, k, gate, valid, lengths, kpool, ape, ln_w, ln_b, eps=1e-5, max_pools=None):
    req_start = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    if max_pools is None:
        max_pools = max(max(lengths) // kpool + 1, 1)
    return orc.kpool_compress(k, gate, valid, req_start, kpool, max_pools, ape, ln_w, ln_b, eps,
                              key_fill=0xFFFF)


def _rand_tokens(rng, T, D, sigma=1.0, mean=0.0):
    return W.f32_to_bf16_bits((mean + sigma * rng.standard_normal((T, D))).astype(np.float32))


def test_knorm_is_layernorm_with_bias(orc):
    """mod.rs trap 1: k_norm is nn.LayerNorm (mean-subtracting, with bias).

    With kpool = 1 every pool is one token and its softmax weight is 1, so the
    pooled key is the bf16 k_norm row itself; compare with torch's layer_norm.
    """
    rng = np.random.default_rng(3)
    T, D = 40, 128
    k = _rand_tokens(rng, T, D, sigma=2.0, mean=0.7)        # nonzero mean: RMSNorm would differ
    gate = _rand_tokens(rng, T, D)
    ln_w = W.f32_to_bf16_bits((1 + 0.3 * rng.standard_normal(D)).astype(np.float32))
    ln_b = W.f32_to_bf16_bits((0.5 * rng.standard_normal(D)).astype(np.float32))
    eps = 1e-5
    keys, idx, pv, fv = _compress(orc, k, gate, np.ones(T, np.uint8), [T], 1,
                                  np.zeros((1, D), np.float32), ln_w, ln_b, eps)
    x = torch.from_numpy(bf16_values(k))
    ref = F.layer_norm(x, (D,), torch.from_numpy(bf16_values(ln_w)),
                       torch.from_numpy(bf16_values(ln_b)), eps=float(np.float32(eps)))
    ref_bits = rnd_bf16(orc, ref.numpy())
    assert pv[0, :T].all() and fv[0] == 0
    np.testing.assert_array_equal(keys[0, :T], ref_bits)
    # single-row entry point agrees with the pooled path
    np.testing.assert_array_equal(orc.layernorm_row(k[5], ln_w, ln_b, eps), ref_bits[5])


def test_knorm_closed_form(orc):
    """Closed form: with w = 1, b = beta the output has mean beta and variance s2/(s2+eps)."""
    rng = np.random.default_rng(4)
    D = 128
    x = _rand_tokens(rng, 1, D, sigma=3.0, mean=-2.0)[0]
    xv = bf16_values(x)
    s2 = xv.var()
    for eps in (1e-5, 0.5):
        y = bf16_values(orc.layernorm_row(x, W.f32_to_bf16_bits(np.ones(D, np.float32)),
                                          W.f32_to_bf16_bits(np.full(D, 0.25, np.float32)), eps))
        e32 = float(np.float32(eps))
        assert abs(y.mean() - 0.25) < 4e-3
        assert abs(((y - 0.25) ** 2).mean() - s2 / (s2 + e32)) < 8e-3


# --------------------------------------------------------------------------- a3 kpool_compress
def _kn_rows(orc, k, ln_w, ln_b, eps=1e-5):
    return np.stack([orc.layernorm_row(r, ln_w, ln_b, eps) for r in k])


def _setup(rng, T, D=128):
    k = _rand_tokens(rng, T, D)
    gate = _rand_tokens(rng, T, D)
    ln_w = W.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(D)).astype(np.float32))
    ln_b = W.f32_to_bf16_bits((0.1 * rng.standard_normal(D)).astype(np.float32))
    return k, gate, ln_w, ln_b


def test_compress_softmax_over_slots_vs_library(orc):
    """mod.rs trap 2: softmax over the pool-slot axis, per channel (torch.softmax, dim=slot)."""
    rng = np.random.default_rng(5)
    D, kp, T = 128, 4, 4 * 9
    k, gate, ln_w, ln_b = _setup(rng, T, D)
    ape = (0.5 * rng.standard_normal((kp, D))).astype(np.float32)
    keys, idx, pv, fv = _compress(orc, k, gate, np.ones(T, np.uint8), [T], kp, ape, ln_w, ln_b)
    kn = bf16_values(_kn_rows(orc, k, ln_w, ln_b)).reshape(T // kp, kp, D)
    lg = bf16_values(gate).reshape(T // kp, kp, D) + ape.astype(np.float64)[None]
    wts = torch.softmax(torch.from_numpy(lg), dim=1).numpy()
    ref = rnd_bf16(orc, (wts * kn).sum(axis=1))
    assert pv[0, :T // kp].all()
    np.testing.assert_array_equal(keys[0, :T // kp], ref)


def test_compress_uniform_gate_gives_mean(orc):
    """Equal logits on every slot: weights 1/kpool, pooled key = mean of the k_norm rows.

    kpool 4 keeps the weights (1/4) and the weighted sum exact in binary64, so
    the comparison is exact even where the mean sits on a bf16 tie.
    """
    rng = np.random.default_rng(6)
    D, kp, T = 128, 4, 4 * 5
    k, _, ln_w, ln_b = _setup(rng, T, D)
    gate = np.tile(_rand_tokens(rng, 1, D), (T, 1))              # same logits on every token
    keys, *_ = _compress(orc, k, gate, np.ones(T, np.uint8), [T], kp,
                         np.zeros((kp, D), np.float32), ln_w, ln_b)
    kn = bf16_values(_kn_rows(orc, k, ln_w, ln_b)).reshape(T // kp, kp, D)
    np.testing.assert_array_equal(keys[0, :T // kp], rnd_bf16(orc, kn.mean(axis=1)))


def test_compress_dominant_slot_and_ape(orc):
    """A slot whose ape logit dominates takes all the weight: pooled key = that slot's row."""
    rng = np.random.default_rng(7)
    D, kp, T = 128, 4, 16
    k, gate, ln_w, ln_b = _setup(rng, T, D)
    kn = _kn_rows(orc, k, ln_w, ln_b).reshape(T // kp, kp, D)
    for s_star in range(kp):
        ape = np.zeros((kp, D), np.float32)
        ape[s_star] = 1000.0
        keys, *_ = _compress(orc, k, gate, np.ones(T, np.uint8), [T], kp, ape, ln_w, ln_b)
        np.testing.assert_array_equal(keys[0, :T // kp], kn[:, s_star])


def test_compress_weights_sum_to_one(orc):
    """mod.rs trap 2 invariant: the slot weights of each channel sum to 1.

    If every slot of a pool holds the same token, sum_s w_s * kn = kn exactly
    when the weights sum to 1, whatever the logits are.
    """
    rng = np.random.default_rng(8)
    D, kp = 128, 8
    row = _rand_tokens(rng, 1, D)
    k = np.tile(row, (kp * 3, 1))
    gate = _rand_tokens(rng, kp * 3, D, sigma=3.0)
    ln_w, ln_b = _setup(rng, 1, D)[2:]
    ape = (rng.standard_normal((kp, D))).astype(np.float32)
    keys, *_ = _compress(orc, k, gate, np.ones(kp * 3, np.uint8), [kp * 3], kp, ape, ln_w, ln_b)
    kn = orc.layernorm_row(row[0], ln_w, ln_b, 1e-5)
    for p in range(3):
        np.testing.assert_array_equal(keys[0, p], kn)


def test_compress_left_padding_and_partial_pool(orc):
    """mod.rs traps 3-4: pools start at the first valid token; a partial tail pool is dropped."""
    rng = np.random.default_rng(9)
    D, kp = 128, 4
    lengths = [37, 29, 6, 4]
    pads = [5, 0, 3, 4]          # request 3 is all padding
    T = sum(lengths)
    k, gate, ln_w, ln_b = _setup(rng, T, D)
    valid = np.ones(T, np.uint8)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    for b, p in enumerate(pads):
        valid[starts[b]:starts[b] + p] = 0
    ape = (0.1 * rng.standard_normal((kp, D))).astype(np.float32)
    P = 12
    keys, idx, pv, fv = _compress(orc, k, gate, valid, lengths, kp, ape, ln_w, ln_b, max_pools=P)
    assert list(fv) == pads
    for b in range(len(lengths)):
        n_valid = (lengths[b] - pads[b]) // kp
        assert pv[b].sum() == n_valid and pv[b, :n_valid].all()
        for p in range(n_valid):
            assert list(idx[b, p]) == [pads[b] + p * kp + s for s in range(kp)]
        assert (idx[b, n_valid:] == -1).all()
        # rows past the span are not written
        assert (keys[b, n_valid:] == 0xFFFF).all()
    # changing the padding tokens' values changes nothing
    k2, gate2 = k.copy(), gate.copy()
    for b, p in enumerate(pads):
        k2[starts[b]:starts[b] + p] = _rand_tokens(rng, p, D)
        gate2[starts[b]:starts[b] + p] = _rand_tokens(rng, p, D)
    keys2, idx2, pv2, fv2 = _compress(orc, k2, gate2, valid, lengths, kp, ape, ln_w, ln_b,
                                      max_pools=P)
    np.testing.assert_array_equal(keys2, keys)
    # and so does the trailing partial pool's content
    k3 = k.copy()
    for b in range(len(lengths)):
        tail0 = starts[b] + pads[b] + ((lengths[b] - pads[b]) // kp) * kp
        k3[tail0:starts[b + 1]] = _rand_tokens(rng, starts[b + 1] - tail0, D)
    keys3, *_ = _compress(orc, k3, gate, valid, lengths, kp, ape, ln_w, ln_b, max_pools=P)
    np.testing.assert_array_equal(keys3, keys)


def test_compress_hole_invalidates_only_its_pool(orc):
    """mod.rs trap 4: a pool counts only if every slot is valid; its key is zero."""
    rng = np.random.default_rng(10)
    D, kp, T = 128, 4, 32
    k, gate, ln_w, ln_b = _setup(rng, T, D)
    valid = np.ones(T, np.uint8)
    valid[0] = 0          # f = 1
    valid[1 + 4 * 3 + 2] = 0      # slot 2 of pool 3
    keys, idx, pv, fv = _compress(orc, k, gate, valid, [T], kp, np.zeros((kp, D), np.float32),
                                  ln_w, ln_b, max_pools=10)
    assert fv[0] == 1
    assert list(pv[0]) == [1, 1, 1, 0, 1, 1, 1, 0, 0, 0]
    assert (keys[0, 3] == 0).all() and (idx[0, 3] == -1).all()
    assert list(idx[0, 4]) == [17, 18, 19, 20]


# --------------------------------------------------------------------------- a4 index_scores
def _scores(orc, q_idx, gate_w, keys, pv, fv, kpool, q_pos, q_req=None):
    Q = q_idx.shape[0]
    q_req = np.zeros(Q, np.int32) if q_req is None else q_req
    return orc.index_scores(q_idx, gate_w, q_req, np.asarray(q_pos, np.int32), keys, pv, fv, kpool)


def test_scores_single_head_is_relu_dot(orc):
    rng = np.random.default_rng(12)
    D, P = 128, 20
    keys = _rand_tokens(rng, P, D)[None]
    q = _rand_tokens(rng, 1, D)[None]
    pv = np.ones((1, P), np.uint8)
    s, c = _scores(orc, q, np.ones((1, 1), np.float32), keys, pv, np.zeros(1, np.int32), 1,
                   [P - 1])
    dots = bf16_values(keys[0]) @ bf16_values(q[0, 0])
    np.testing.assert_array_equal(s[0], np.maximum(dots, 0).astype(np.float32))
    assert (dots < 0).any() and (s[0] == 0).sum() == (dots <= 0).sum()


def test_scores_head_gate_weights_and_sign(orc):
    rng = np.random.default_rng(13)
    D, P, H = 128, 24, 16
    keys = _rand_tokens(rng, P, D)[None]
    q = _rand_tokens(rng, 1, H * D).reshape(1, H, D)
    g = rng.standard_normal((1, H)).astype(np.float32)
    pv = np.ones((1, P), np.uint8)
    fv = np.zeros(1, np.int32)
    s, _ = _scores(orc, q, g, keys, pv, fv, 1, [P - 1])
    dots = np.einsum("hc,pc->hp", bf16_values(q[0]), bf16_values(keys[0]))
    ref = (g[0].astype(np.float64)[:, None] * np.maximum(dots, 0)).sum(0)
    np.testing.assert_allclose(s[0], ref.astype(np.float32), rtol=1e-6, atol=1e-6)
    s0, _ = _scores(orc, q, np.zeros_like(g), keys, pv, fv, 1, [P - 1])
    assert (s0 == 0).all()
    sneg, _ = _scores(orc, q, -g, keys, pv, fv, 1, [P - 1])
    np.testing.assert_array_equal(sneg, -s)


def test_scores_candidate_rule(orc):
    """Candidates: valid pools whose last token is at or before the query position; -inf else."""
    rng = np.random.default_rng(14)
    D, kp, P = 128, 4, 8
    keys = _rand_tokens(rng, P, D)[None]
    pv = np.ones((1, P), np.uint8)
    pv[0, 2] = 0
    fv = np.array([3], np.int32)
    q = _rand_tokens(rng, 1, 16 * D).reshape(1, 16, D)
    g = np.ones((1, 16), np.float32)
    # pool p's last token = 3 + 4p + 3
    for q_pos, n_ok in [(3 + 4 * 5 + 3, 6), (3 + 4 * 5 + 2, 5), (2, 0), (1000, 8)]:
        s, c = _scores(orc, q, g, keys, pv, fv, kp, [q_pos])
        expect = np.array([(p < n_ok) and p != 2 for p in range(P)])
        np.testing.assert_array_equal(c[0].astype(bool), expect)
        assert np.isneginf(s[0][~expect]).all() and np.isfinite(s[0][expect]).all()


# --------------------------------------------------------------------------- a5/a6 top-k + expand
def _pool_idx(P, kp, f=0):
    return np.array([[[f + p * kp + s for s in range(kp)] for p in range(P)]], np.int32)


def test_topk_vs_sorted_with_ties(orc):
    rng = np.random.default_rng(15)
    Q, P, kp, K = 6, 300, 4, 64
    scores = np.round(rng.standard_normal((Q, P)) * 3).astype(np.float32)   # many ties
    cand = (rng.random((Q, P)) < 0.8).astype(np.uint8)
    cand[5, :] = 0
    cand[5, :10] = 1            # fewer candidates than K
    scores[~cand.astype(bool)] = -np.inf
    scores[0, 7] = np.float32(50.0)
    cand[0, 7] = 0              # a non-candidate never ranks, whatever its score
    pidx = np.repeat(_pool_idx(P, kp, f=2), 1, axis=0)
    top, ids = orc.topk_expand(scores, cand, pidx, np.zeros(Q, np.int32), K)
    for q in range(Q):
        cands = [p for p in range(P) if cand[q, p]]
        ranked = sorted(cands, key=lambda p: (-float(scores[q, p]), p))[:K]
        chosen = sorted(ranked)              # the selected set, listed by pool id
        expect = chosen + [-1] * (K - len(chosen))
        assert list(top[q]) == expect
        exp_ids = sum(([2 + p * kp + s for s in range(kp)] if p >= 0 else [-1] * kp
                       for p in expect), [])
        assert list(ids[q]) == exp_ids
    assert 7 not in top[0]


def test_topk_all_equal_and_width(orc):
    Q, P, kp, K = 2, 50, 3, 16
    scores = np.zeros((Q, P), np.float32)
    cand = np.ones((Q, P), np.uint8)
    top, ids = orc.topk_expand(scores, cand, _pool_idx(P, kp), np.zeros(Q, np.int32), K)
    assert ids.shape == (Q, K * kp)                    # out_width = select_k * kpool
    assert (top == np.arange(K)).all()                 # ties -> lowest pool id
    cand[:] = 0
    top, ids = orc.topk_expand(scores, cand, _pool_idx(P, kp), np.zeros(Q, np.int32), K)
    assert (top == -1).all() and (ids == -1).all()     # sentinel written in full


def test_topk_nan_ranks_as_neg_inf(orc):
    scores = np.array([[np.nan, -np.inf, 1.0, -5.0, 0.5]], np.float32)
    cand = np.ones((1, 5), np.uint8)
    # ranking 2 > 4 > 3 > {0 (NaN as -inf), 1 (-inf)}, tie -> lower id: 0 before 1
    top, _ = orc.topk_expand(scores, cand, _pool_idx(5, 1), np.zeros(1, np.int32), 4)
    assert list(top[0]) == [0, 2, 3, 4]
    top, _ = orc.topk_expand(scores, cand, _pool_idx(5, 1), np.zeros(1, np.int32), 3)
    assert list(top[0]) == [2, 3, 4]


# --------------------------------------------------------------------------- a7 sparse MLA
def _mla(orc, q, kv, ids, scale, lengths=None):
    T = kv.shape[0]
    lengths = [T] if lengths is None else lengths
    rs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return orc.sparse_mla(q, kv, rs, np.zeros(q.shape[0], np.int32), np.asarray(ids, np.int32),
                          scale)


def test_mla_single_token_returns_its_row(orc):
    rng = np.random.default_rng(16)
    T, L, Hm = 30, 512, 4
    kv = _rand_tokens(rng, T, L)
    q = _rand_tokens(rng, Hm, L).reshape(1, Hm, L)
    out, lse = _mla(orc, q, kv, [[-1, 17, -1, -1]], 0.05)
    for h in range(Hm):
        np.testing.assert_array_equal(out[0, h], kv[17])
        z = 0.05 * float(bf16_values(q[0, h]) @ bf16_values(kv[17]))
        assert abs(lse[0, h] - z) <= 1e-6 * max(1, abs(z))


def test_mla_zero_query_is_mean_of_selected(orc):
    rng = np.random.default_rng(17)
    T, L = 40, 512
    kv = _rand_tokens(rng, T, L)
    q = np.zeros((1, 2, L), np.uint16)
    sel = [3, 9, 33, 39]          # 4 tokens: weights 1/4 and their sums are exact in binary64
    out, lse = _mla(orc, q, kv, [sel + [-1, -1]], 0.1)
    np.testing.assert_array_equal(out[0, 0], rnd_bf16(orc, bf16_values(kv[sel]).mean(0)))
    assert abs(lse[0, 0] - math.log(len(sel))) < 1e-6


def test_mla_set_semantics(orc):
    """mod.rs MASKED_ATTN_MAX_KEYS doc: a set mask; duplicates collapse, order is irrelevant."""
    rng = np.random.default_rng(18)
    T, L, Hm = 64, 512, 3
    kv = _rand_tokens(rng, T, L)
    q = _rand_tokens(rng, Hm, L).reshape(1, Hm, L)
    sel = [5, 60, 2, 33, 34, 35]
    a, la = _mla(orc, q, kv, [sel + [-1] * 4], 0.044)
    b, lb = _mla(orc, q, kv, [list(reversed(sel)) + [5, 5, 33, -1]], 0.044)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    e, le = _mla(orc, q, kv, [[-1] * 10], 0.044)
    assert (e == 0).all() and np.isneginf(le).all()


def test_mla_vs_library_sdpa(orc):
    """Dense masked attention with torch SDPA (fp64, boolean mask) on a tiny case."""
    rng = np.random.default_rng(19)
    lengths = [50, 70]
    T, L, Hm, Wd = sum(lengths), 512, 4, 24
    kv = _rand_tokens(rng, T, L)
    q = _rand_tokens(rng, 2 * Hm, L).reshape(2, Hm, L)
    ids = np.full((2, Wd), -1, np.int32)
    ids[0, :20] = rng.choice(50, 20, replace=False)
    ids[1, :Wd] = rng.choice(70, Wd, replace=False)
    rs = np.array([0, 50, 120], np.int32)
    scale = float(np.float32(1 / math.sqrt(L)))
    out, lse = orc.sparse_mla(q, kv, rs, np.array([0, 1], np.int32), ids, scale)
    kvf = bf16_values(kv)
    for i in range(2):
        rows = kvf[rs[i]:rs[i + 1]]
        mask = np.zeros(lengths[i], bool)
        mask[ids[i][ids[i] >= 0]] = True
        qq = torch.from_numpy(bf16_values(q[i]))[None]          # [1, Hm, L]
        kk = torch.from_numpy(rows)[None, None].expand(1, Hm, -1, -1)
        o = F.scaled_dot_product_attention(qq[:, :, None], kk, kk,
                                           attn_mask=torch.from_numpy(mask)[None, None, None],
                                           scale=scale)[0, :, 0]
        np.testing.assert_array_equal(out[i], rnd_bf16(orc, o.numpy()))
        z = scale * (bf16_values(q[i]) @ rows[mask].T)
        np.testing.assert_allclose(lse[i], torch.logsumexp(torch.from_numpy(z), -1).numpy(),
                                   rtol=1e-6, atol=1e-6)


def test_mla_physical_rows_are_request_relative(orc):
    """Token ids are logical per request; physical row = req_start[b] + id."""
    rng = np.random.default_rng(20)
    lengths = [10, 10]
    kv = _rand_tokens(rng, 20, 512)
    q = np.zeros((1, 1, 512), np.uint16)
    rs = np.array([0, 10, 20], np.int32)
    out, _ = orc.sparse_mla(q, kv, rs, np.array([1], np.int32), np.array([[4]], np.int32), 0.1)
    np.testing.assert_array_equal(out[0, 0], kv[14])


def test_indexer_store_places_rows_by_request_and_position(orc):
    """Stored rows land at req_start[b] + pos, marked valid; out-of-range rows are dropped."""
    req_start = np.array([0, 3, 3, 7], np.int32)          # request 1 is empty
    k = np.zeros((7, 2), np.uint16)
    gate = np.zeros((7, 2), np.uint16)
    valid = np.zeros(7, np.uint8)
    k_new = np.array([[1, 2], [3, 4], [5, 6], [7, 8], [9, 10]], np.uint16)
    g_new = k_new + 100
    tok_req = np.array([0, 2, 1, 2, 3])                  # request 1 has no row 0; request 3 is none
    tok_pos = np.array([2, 0, 0, 4, 0])                  # position 4 is past request 2's 4 rows
    k2, g2, v2 = orc.indexer_store(k, gate, valid, req_start, k_new, g_new, None, tok_req, tok_pos)
    want_k = np.zeros((7, 2), np.uint16)
    want_k[2] = [1, 2]
    want_k[3] = [3, 4]
    np.testing.assert_array_equal(k2, want_k)
    np.testing.assert_array_equal(g2[[2, 3]], [[101, 102], [103, 104]])
    assert g2[[0, 1, 4, 5, 6]].sum() == 0
    np.testing.assert_array_equal(v2, [0, 0, 1, 1, 0, 0, 0])
    assert valid.sum() == 0 and k.sum() == 0               # inputs are not modified
    # an explicit validity byte is stored as given (nonzero -> 1)
    _, _, v3 = orc.indexer_store(k, gate, np.ones(7, np.uint8), req_start, k_new[:2], g_new[:2],
                                 np.array([0, 7], np.uint8), tok_req[:2], tok_pos[:2])
    np.testing.assert_array_equal(v3, [1, 1, 0, 1, 1, 1, 1])


def test_compress_after_store_only_changes_pools_of_new_tokens(orc):
    """Appending tokens to a capacity-sized request changes only the pools that hold them.

    This is what lets the incremental update recompute those pools alone
    (pooled keys of a pool depend only on its own kpool token rows, given f_b).
    """
    rng = np.random.default_rng(11)
    kp, cap = 4, 40
    req_start = np.array([0, cap], np.int32)
    k = rng.integers(0x3C00, 0x4000, size=(cap, 128)).astype(np.uint16)     # bf16 values in [1, 2)
    gate = rng.integers(0x3C00, 0x4000, size=(cap, 128)).astype(np.uint16)
    valid = np.zeros(cap, np.uint8)
    valid[3:21] = 1                                        # f = 3, tokens 3..20 present
    ape = rng.standard_normal((kp, 128)).astype(np.float32) * np.float32(0.02)
    ln_w = np.full(128, 0x3F80, np.uint16)
    ln_b = np.zeros(128, np.uint16)
    before = orc.kpool_compress(k, gate, valid, req_start, kp, 10, ape, ln_w, ln_b, 1e-5)
    k2, g2, v2 = orc.indexer_store(k, gate, valid, req_start, k[21:24] ^ 1, gate[21:24], None,
                                   [0, 0, 0], [21, 22, 23])
    after = orc.kpool_compress(k2, g2, v2, req_start, kp, 10, ape, ln_w, ln_b, 1e-5)
    assert before[3][0] == after[3][0] == 3
    # pools 0..3 (tokens 3..18) unchanged; pool 4 (tokens 19..22) and 5 (23..26) hold new tokens
    for a, b in zip(before[:3], after[:3]):
        np.testing.assert_array_equal(a[0, :4], b[0, :4])
        np.testing.assert_array_equal(a[0, 6:], b[0, 6:])
    assert before[2][0, 4] == 0 and after[2][0, 4] == 1    # pool 4 complete now
    assert after[2][0, 5] == 0                             # pool 5 still lacks tokens 24..26
    assert not np.array_equal(before[0][0, 4], after[0][0, 4])


def test_tail_slots_hold_the_trailing_partial_pool(orc):
    """Tail slots: the tokens after the query's last complete pool, up to q_pos."""
    req_start = np.array([0, 20, 30, 30], np.int32)         # request 2 is empty
    valid = np.ones(30, np.uint8)
    valid[0:3] = 0                                          # request 0: f = 3
    valid[20 + 8] = 0                                       # request 1: a hole at token 8
    first_valid = np.array([3, 0, 0], np.int32)
    kp = 4
    q_req = np.array([0, 0, 0, 0, 1, 1, 2, 7])
    q_pos = np.array([9, 10, 14, 2, 9, 5, 0, 3])
    got = orc.tail_slots(q_req, q_pos, first_valid, valid, req_start, kp)
    want = np.array([
        [7, 8, 9],      # tokens 3..6 form pool 0; 7, 8, 9 trail
        [-1, -1, -1],   # 3..10 are two complete pools: nothing trails
        [-1, -1, -1],   # 3..14 three complete pools
        [-1, -1, -1],   # q_pos before the first valid token
        [-1, 9, -1],    # pools 0..3, 4..7; 8 (a hole) and 9 trail: the hole's slot is -1
        [4, 5, -1],
        [-1, -1, -1],   # empty request: f = T = 0 but token 0 does not exist
        [-1, -1, -1],   # request out of range
    ], np.int32)
    np.testing.assert_array_equal(got, want)
    # kpool 1: no tail slots at all
    assert orc.tail_slots(q_req, q_pos, first_valid, valid, req_start, 1).shape == (8, 0)
    # the tail never repeats a token of a candidate pool: candidates end at or before q_pos
    rng = np.random.default_rng(3)
    for _ in range(50):
        kp = int(rng.integers(2, 9))
        f = int(rng.integers(0, 5))
        qp = int(rng.integers(f, 60))
        t = orc.tail_slots([0], [qp], [f], np.ones(64, np.uint8), [0, 64], kp)[0]
        last_cand_end = f + ((qp - f + 1) // kp) * kp - 1   # last token of the last candidate pool
        ids = t[t >= 0]
        assert (ids > last_cand_end).all() and (ids <= qp).all()
        assert len(ids) == (qp - f + 1) % kp


def test_paged_mla_single_token_reads_its_page_row(orc):
    """One selected token: out is its latent row, wherever its page sits."""
    rng = np.random.default_rng(5)
    L, page = 512, 2
    kv = W.f32_to_bf16_bits(rng.standard_normal((8, L), dtype=np.float32))   # 4 pages
    block_table = np.array([[3, 0, -1], [1, 2, -1]], np.int32)   # request 0: pages 3, 0
    seq_len = np.array([4, 3], np.int32)
    q = W.f32_to_bf16_bits(rng.standard_normal((3, 16, L), dtype=np.float32))
    q_req = np.array([0, 0, 1])
    ids = np.array([[2, -1], [1, -1], [2, 7]], np.int32)       # 7 is past request 1's tokens
    out, lse = orc.sparse_mla_paged(q, kv, block_table, page, seq_len, q_req, ids, 0.05)
    # request 0 token 2 -> page 0 row 0 = cache row 0; token 1 -> page 3 row 1 = cache row 7;
    # request 1 token 2 -> page 2 row 0 = cache row 4
    for i, row in enumerate([0, 7, 4]):
        for h in range(16):
            np.testing.assert_array_equal(out[i, h], kv[row])
    # a token on a missing page is dropped: nothing valid -> out 0, lse -inf
    out2, lse2 = orc.sparse_mla_paged(q[:1], kv, np.array([[-1, 0]], np.int32), page, [4], [0],
                                      np.array([[0, 1]], np.int32), 0.05)
    assert (out2 == 0).all() and np.isneginf(lse2).all()


def test_paged_mla_is_invariant_to_page_placement(orc):
    """Moving the pages of a cache (and its table with them) leaves the result unchanged."""
    rng = np.random.default_rng(9)
    L, page, T = 512, 4, 22
    n_pages = (T + page - 1) // page                              # 6 pages
    kv_c = W.f32_to_bf16_bits(rng.standard_normal((T, L), dtype=np.float32))
    perm = rng.permutation(10)[:n_pages]                         # 6 of 10 physical pages
    pool = np.zeros((10 * page, L), np.uint16)
    for pi in range(n_pages):
        rows = kv_c[pi * page:(pi + 1) * page]
        pool[perm[pi] * page:perm[pi] * page + len(rows)] = rows
    table = perm[None, :].astype(np.int32)
    q = W.f32_to_bf16_bits(rng.standard_normal((2, 16, L), dtype=np.float32))
    ids = np.array([rng.permutation(T)[:9], rng.permutation(T)[:9]], np.int32)
    a = orc.sparse_mla_paged(q, pool, table, page, [T], [0, 0], ids, 0.06)
    b = orc.sparse_mla(q, kv_c, [0, T], [0, 0], ids, 0.06)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_e4m3_decode_vs_torch_and_definition(orc):
    """Every E4M3 code against torch's float8_e4m3fn and the format's landmarks."""
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([orc.f64_from_e4m3(int(c)) for c in codes])
    lib_vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib_vals)
    assert (np.isnan(mine) == nan).all() and nan.sum() == 2            # S.1111.111 only
    np.testing.assert_array_equal(mine[~nan], lib_vals[~nan])
    assert orc.f64_from_e4m3(0x7E) == 448.0 and orc.f64_from_e4m3(0x01) == 2.0 ** -9
    assert orc.f64_from_e4m3(0x38) == 1.0 and orc.f64_from_e4m3(0xB8) == -1.0


def test_fp8_mla_single_token_and_scale(orc):
    """One selected token: out = bf16(kv_scale * decoded row); the scale enters the logits."""
    rng = np.random.default_rng(12)
    L = 512
    kv8 = rng.integers(0, 256, size=(5, L)).astype(np.uint8)
    kv8[(kv8 & 0x7F) == 0x7F] = 0x3C                                    # no NaN codes
    q = W.f32_to_bf16_bits(rng.standard_normal((2, 16, L), dtype=np.float32))
    ids = np.array([[3, -1], [1, 4]], np.int32)
    out, lse = orc.sparse_mla_fp8(q, kv8, 0.5, [0, 5], [0, 0], ids, 0.01)
    dec = np.array([[orc.f64_from_e4m3(int(c)) for c in row] for row in kv8])
    want = np.array([orc.bf16_from_f64(0.5 * v) for v in dec[3]], np.uint16)
    for h in range(16):        # as values: a sum that starts at +0 turns a -0 row entry into +0
        np.testing.assert_array_equal(W.bf16_bits_to_f32(out[0, h]), W.bf16_bits_to_f32(want))
    # a power-of-two scale is exact, so the fp8 result equals the bf16 result on the
    # decoded-and-scaled cache (each scaled value is a bf16 value)
    kv_bf16 = np.array([[orc.bf16_from_f64(0.5 * v) for v in row] for row in dec], np.uint16)
    out_b, lse_b = orc.sparse_mla(q, kv_bf16, [0, 5], [0, 0], ids, 0.01)
    np.testing.assert_array_equal(out, out_b)
    np.testing.assert_array_equal(lse, lse_b)
