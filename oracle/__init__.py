"""CPU oracle of the DSA decode path (numpy front end over oracle/dsa_oracle.c).

TEST INFRASTRUCTURE ONLY. The tests, the package smoke check and the bench's
CPU-baseline leg are the only callers; the product path never imports this
package, and it imports nothing from the product package. Each function below
is the plain definition of one stage, computed in binary64 and rounded once to
the stage's storage type; the docstrings of dsa_oracle.c give the definitions
and cite the page passages they follow.

bf16 arrays are numpy uint16 arrays holding bf16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        L.orc_bf16_from_f64.argtypes = [D]
        L.orc_bf16_from_f64.restype = ctypes.c_uint16
        L.orc_f64_from_bf16.argtypes = [ctypes.c_uint16]
        L.orc_f64_from_bf16.restype = D
        L.orc_head_gate.argtypes = [P, P, P, I, I, I, I]
        L.orc_layernorm_row.argtypes = [P, P, P, D, I, P]
        L.orc_kpool_compress.argtypes = [P, P, P, P, I, I, I, I, P, P, P, D, P, P, P, P, I]
        L.orc_index_scores.argtypes = [P, P, P, P, I, I, I, P, P, P, I, I, I, P, P, I]
        L.orc_topk_expand.argtypes = [P, P, P, P, I, I, I, I, I, P, P, I]
        L.orc_sparse_mla.argtypes = [P, P, P, P, P, I, I, I, I, I, D, P, P, I]
        L.orc_sparse_mla_fp8.argtypes = [P, P, D, P, P, P, I, I, I, I, I, D, P, P, I]
        L.orc_f64_from_e4m3.argtypes = [ctypes.c_uint8]
        L.orc_f64_from_e4m3.restype = D
        for f in ("orc_head_gate", "orc_layernorm_row", "orc_kpool_compress",
                  "orc_index_scores", "orc_topk_expand", "orc_sparse_mla", "orc_sparse_mla_fp8"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"oracle {name}: malformed arguments (status {rc})")


def default_threads() -> int:
    return int(os.environ.get("DSA_ORACLE_THREADS", "0"))


def bf16_from_f64(x: float) -> int:
    return int(lib().orc_bf16_from_f64(float(x)))


def f64_from_e4m3(code: int) -> float:
    return float(lib().orc_f64_from_e4m3(int(code)))


def f64_from_bf16(bits: int) -> float:
    return float(lib().orc_f64_from_bf16(int(bits)))


def head_gate(hidden: np.ndarray, w: np.ndarray, threads: int = 0) -> np.ndarray:
    hidden = _c(hidden, np.float32)
    w = _c(w, np.float32)
    M, K = hidden.shape
    K2, N = w.shape
    assert K == K2
    out = np.empty((M, N), dtype=np.float32)
    _check(lib().orc_head_gate(_p(hidden), _p(w), _p(out), M, K, N, threads or default_threads()),
           "head_gate")
    return out


def layernorm_row(x: np.ndarray, ln_w: np.ndarray, ln_b: np.ndarray, eps: float) -> np.ndarray:
    x = _c(x, np.uint16)
    ln_w = _c(ln_w, np.uint16)
    ln_b = _c(ln_b, np.uint16)
    D = x.shape[-1]
    out = np.empty(D, dtype=np.uint16)
    _check(lib().orc_layernorm_row(_p(x), _p(ln_w), _p(ln_b), float(np.float32(eps)), D, _p(out)),
           "layernorm_row")
    return out


def kpool_compress(k, gate, valid, req_start, kpool: int, max_pools: int, ape, ln_w, ln_b,
                   eps: float, threads: int = 0, key_fill: int = 0):
    """Returns (pool_keys [B,P,D] u16, pool_idx [B,P,k] i32, pool_valid [B,P] u8, first_valid [B] i32).

    Rows of pool_keys that the stage does not write keep ``key_fill``.
    """
    k = _c(k, np.uint16)
    gate = _c(gate, np.uint16)
    valid = _c(valid, np.uint8)
    req_start = _c(req_start, np.int32)
    ape = _c(ape, np.float32)
    ln_w = _c(ln_w, np.uint16)
    ln_b = _c(ln_b, np.uint16)
    B = req_start.shape[0] - 1
    D = k.shape[1]
    assert ape.shape == (kpool, D)
    keys = np.full((B, max_pools, D), key_fill, dtype=np.uint16)
    idx = np.empty((B, max_pools, kpool), dtype=np.int32)
    pv = np.empty((B, max_pools), dtype=np.uint8)
    fv = np.empty(B, dtype=np.int32)
    _check(lib().orc_kpool_compress(_p(k), _p(gate), _p(valid), _p(req_start), B, D, kpool,
                                    max_pools, _p(ape), _p(ln_w), _p(ln_b),
                                    float(np.float32(eps)), _p(keys), _p(idx), _p(pv), _p(fv),
                                    threads or default_threads()), "kpool_compress")
    return keys, idx, pv, fv


def indexer_store(k, gate, valid, req_start, k_new, gate_new, valid_new, tok_req, tok_pos):
    """The indexer cache after a step's new rows are stored: copies of (k, gate, valid).

    "spark_model/layers/glm5next_dsa/mod.rs", Glm5NextDsaKernels::indexer_store:
    each staged row goes to the cache row of its request at its position, and
    that token is marked valid. A row whose request or position falls outside
    the cache is not stored (the plainest reading where the page says nothing
    about them); valid_new None marks every stored token valid.
    """
    k, gate, valid = np.array(k, np.uint16), np.array(gate, np.uint16), np.array(valid, np.uint8)
    req_start = np.asarray(req_start, np.int64)
    B = req_start.shape[0] - 1
    for i in range(len(tok_req)):
        b, pos = int(tok_req[i]), int(tok_pos[i])
        if not (0 <= b < B):
            continue
        if not (0 <= pos < req_start[b + 1] - req_start[b]):
            continue
        row = req_start[b] + pos
        k[row] = k_new[i]
        gate[row] = gate_new[i]
        valid[row] = 1 if valid_new is None or valid_new[i] != 0 else 0
    return k, gate, valid


def index_scores(q_idx, gate_w, q_req, q_pos, pool_keys, pool_valid, first_valid, kpool: int,
                 threads: int = 0):
    """Returns (scores [Q,P] f32, cand [Q,P] u8)."""
    q_idx = _c(q_idx, np.uint16)
    gate_w = _c(gate_w, np.float32)
    q_req = _c(q_req, np.int32)
    q_pos = _c(q_pos, np.int32)
    pool_keys = _c(pool_keys, np.uint16)
    pool_valid = _c(pool_valid, np.uint8)
    first_valid = _c(first_valid, np.int32)
    Q, H, D = q_idx.shape
    B, P = pool_valid.shape
    scores = np.empty((Q, P), dtype=np.float32)
    cand = np.empty((Q, P), dtype=np.uint8)
    _check(lib().orc_index_scores(_p(q_idx), _p(gate_w), _p(q_req), _p(q_pos), Q, H, D,
                                  _p(pool_keys), _p(pool_valid), _p(first_valid), B, kpool, P,
                                  _p(scores), _p(cand), threads or default_threads()),
           "index_scores")
    return scores, cand


def topk_expand(scores, cand, pool_idx, q_req, select_k: int, threads: int = 0):
    """Returns (top_pools [Q,select_k] i32, token_ids [Q,select_k*kpool] i32)."""
    scores = _c(scores, np.float32)
    cand = _c(cand, np.uint8)
    pool_idx = _c(pool_idx, np.int32)
    q_req = _c(q_req, np.int32)
    Q, P = scores.shape
    B, P2, kpool = pool_idx.shape
    assert P == P2
    top = np.empty((Q, select_k), dtype=np.int32)
    ids = np.empty((Q, select_k * kpool), dtype=np.int32)
    _check(lib().orc_topk_expand(_p(scores), _p(cand), _p(pool_idx), _p(q_req), Q, B, P, kpool,
                                 select_k, _p(top), _p(ids), threads or default_threads()),
           "topk_expand")
    return top, ids


def tail_slots(q_req, q_pos, first_valid, valid, req_start, kpool: int) -> np.ndarray:
    """The kpool - 1 tail slots of each query's index row under always_select_tail.

    "spark_model/layers/glm5next_dsa/mod.rs", Glm5NextDsaConfig::out_width: the
    tail adds kpool - 1 slots to the row (the step tap names them idx.tail_slot).
    Reading: they hold the query's trailing partial pool -- the tokens after its
    last complete pool up to and including q_pos, counted on the pool grid that
    starts at the request's first valid token -- in position order, a token that
    is missing or not valid as -1, and -1 past them.
    """
    req_start = np.asarray(req_start, np.int64)
    B = req_start.shape[0] - 1
    Q = len(q_req)
    out = np.full((Q, max(kpool - 1, 0)), -1, dtype=np.int32)
    for q in range(Q):
        b = int(q_req[q])
        if not (0 <= b < B):
            continue
        f, qp = int(first_valid[b]), int(q_pos[q])
        T = int(req_start[b + 1] - req_start[b])
        if qp < f:
            continue
        n_tail = (qp - f + 1) % kpool          # tokens past the last complete pool
        for s in range(n_tail):
            t = qp + 1 - n_tail + s
            if 0 <= t < T and valid[req_start[b] + t] != 0:
                out[q, s] = t
    return out


def sparse_mla(q, kv, req_start, q_req, token_ids, sm_scale: float, threads: int = 0):
    """Returns (out [Q,Hm,L] u16 bf16 bits, lse [Q,Hm] f32)."""
    q = _c(q, np.uint16)
    kv = _c(kv, np.uint16)
    req_start = _c(req_start, np.int32)
    q_req = _c(q_req, np.int32)
    token_ids = _c(token_ids, np.int32)
    Q, Hm, L = q.shape
    W = token_ids.shape[1]
    B = req_start.shape[0] - 1
    out = np.empty((Q, Hm, L), dtype=np.uint16)
    lse = np.empty((Q, Hm), dtype=np.float32)
    _check(lib().orc_sparse_mla(_p(q), _p(kv), _p(req_start), _p(q_req), _p(token_ids), Q, B, Hm,
                                W, L, float(np.float32(sm_scale)), _p(out), _p(lse),
                                threads or default_threads()), "sparse_mla")
    return out, lse


def sparse_mla_fp8(q, kv8, kv_scale: float, req_start, q_req, token_ids, sm_scale: float,
                   threads: int = 0):
    """sparse_mla over an fp8 latent cache: row values kv_scale * E4M3(kv8).

    The pages name an fp8 variant of the paged MLA decode and give no scale
    layout; the reading taken is one fp32 scale for the whole cache.
    """
    q = _c(q, np.uint16)
    kv8 = _c(kv8, np.uint8)
    req_start = _c(req_start, np.int32)
    q_req = _c(q_req, np.int32)
    token_ids = _c(token_ids, np.int32)
    Q, Hm, L = q.shape
    W = token_ids.shape[1]
    B = req_start.shape[0] - 1
    out = np.empty((Q, Hm, L), dtype=np.uint16)
    lse = np.empty((Q, Hm), dtype=np.float32)
    _check(lib().orc_sparse_mla_fp8(_p(q), _p(kv8), float(np.float32(kv_scale)), _p(req_start),
                                    _p(q_req), _p(token_ids), Q, B, Hm, W, L,
                                    float(np.float32(sm_scale)), _p(out), _p(lse),
                                    threads or default_threads()), "sparse_mla_fp8")
    return out, lse


def sparse_mla_paged(q, kv, block_table, page_size: int, seq_len, q_req, token_ids,
                     sm_scale: float, threads: int = 0):
    """Sparse MLA over a block-table paged latent cache: (out, lse) as sparse_mla.

    "spark_model/layers/glm5next_dsa/mod.rs", MASKED_ATTN_MAX_KEYS doc: the serve
    path is the block-table paged MLA decode walking a selected-index row. The
    block table only says where a token's latent row is stored: request b's
    token t is row block_table[b, t // page_size] * page_size + t % page_size.
    Written out as that lookup followed by the contiguous definition: each
    request's rows are copied into a contiguous cache, and an id whose page is
    missing (index past the table, negative block, row past the cache) is
    dropped like -1.
    """
    kv = np.asarray(kv, np.uint16)
    block_table = np.asarray(block_table, np.int64)
    B, max_blocks = block_table.shape
    token_ids = np.array(token_ids, np.int32)
    lengths = [max(int(seq_len[b]), 0) for b in range(B)]
    req_start = np.zeros(B + 1, np.int32)
    req_start[1:] = np.cumsum(lengths)
    flat = np.zeros((int(req_start[-1]), kv.shape[1]), np.uint16)
    present = np.zeros(int(req_start[-1]), bool)
    for b in range(B):
        for t in range(lengths[b]):
            pi = t // page_size
            if pi >= max_blocks or block_table[b, pi] < 0:
                continue
            row = int(block_table[b, pi]) * page_size + t % page_size
            if row >= kv.shape[0]:
                continue
            flat[req_start[b] + t] = kv[row]
            present[req_start[b] + t] = True
    for i in range(token_ids.shape[0]):
        b = int(q_req[i])
        if not (0 <= b < B):
            continue
        for j in range(token_ids.shape[1]):
            t = int(token_ids[i, j])
            if 0 <= t < lengths[b] and not present[req_start[b] + t]:
                token_ids[i, j] = -1
    return sparse_mla(q, flat, req_start, q_req, token_ids, sm_scale, threads)


def pipeline(wl, threads: int = 0, queries: Optional[np.ndarray] = None) -> dict:
    """All stages on a workload's raw inputs (optionally a subset of queries)."""
    qsel = np.arange(wl.Q) if queries is None else np.asarray(queries)
    gate_w = head_gate(wl.hidden[qsel], wl.w_gate, threads)
    keys, idx, pv, fv = kpool_compress(wl.k, wl.gate, wl.valid, wl.req_start, wl.kpool,
                                       wl.max_pools, wl.ape, wl.ln_w, wl.ln_b, wl.eps, threads)
    scores, cand = index_scores(wl.q_idx[qsel], gate_w, wl.q_req[qsel], wl.q_pos[qsel], keys, pv,
                                fv, wl.kpool, threads)
    top, ids = topk_expand(scores, cand, idx, wl.q_req[qsel], wl.select_k, threads)
    out, lse = sparse_mla(wl.q_mla[qsel], wl.kv, wl.req_start, wl.q_req[qsel], ids, wl.sm_scale,
                          threads)
    return dict(gate_w=gate_w, pool_keys=keys, pool_idx=idx, pool_valid=pv, first_valid=fv,
                scores=scores, cand=cand, top_pools=top, token_ids=ids, out=out, lse=lse)
