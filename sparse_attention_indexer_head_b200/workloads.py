"""Seeded synthetic inputs for the DSA decode path.

This module only draws input arrays (shapes, value distributions, padding and
length mixes). It holds none of the path's arithmetic: no normalisation, no
pooling, no scoring, no selection. Both the CUDA path (through the tests and
``bench.py``) and the CPU oracle consume the arrays it returns.

Workloads follow the shapes the GLM-5.3-Flash DSA pages describe:

* head gate ``[M, 4096] x [4096, 16]`` fp32 (page "indexer fp32 head-gate
  split-K", PR description);
* indexer key cache ``[sum T, 128]`` bf16 with per-token compress-gate logits and
  a per-token validity byte, ``kpool`` slots per pool, ``index_topk`` selected
  tokens (page "spark_model/layers/glm5next_dsa/mod.rs", *Shape of the pipeline*
  and ``Glm5NextDsaConfig``);
* NoPE latent cache ``[sum T, 512]`` bf16 (same page, ``kv_cache_dim``).

Notation for distributions: ``N(0, s)`` means a normal with standard deviation
``s``. bf16 arrays are returned as their raw ``uint16`` bit patterns (rounded
to nearest, ties to even, from float32 draws).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

HIDDEN = 4096        # model hidden size feeding the head gate
INDEX_HEADS = 16     # indexer heads (head-gate N)
INDEX_DIM = 128      # indexer head dim (pooled key width)
KV_LORA = 512        # latent width of the NoPE MLA cache


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    flat = x.reshape(-1).view(np.uint32)
    out = np.empty(flat.shape, dtype=np.uint16)
    step = 1 << 22
    for i in range(0, flat.size, step):
        u = flat[i:i + step].astype(np.uint64)
        u += 0x7FFF + ((u >> 16) & 1)
        out[i:i + step] = (u >> 16).astype(np.uint16)
    return out.reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    """One batch of DSA decode/prefill inputs (host arrays)."""

    name: str
    seed: int
    kpool: int
    max_pools: int
    select_k: int
    hm: int                       # MLA heads
    lengths: List[int]            # T_b, tokens cached per request
    pads: List[int]               # left padding per request (invalid tokens)
    q_req: np.ndarray             # [Q] int32 request of each query
    q_pos: np.ndarray             # [Q] int32 position of each query in its request
    hidden: np.ndarray            # [M, 4096] float32 (M == Q)
    w_gate: np.ndarray            # [4096, 16] float32
    q_idx: np.ndarray             # [Q, 16, 128] bf16 bits
    k: np.ndarray                 # [sum T, 128] bf16 bits
    gate: np.ndarray              # [sum T, 128] bf16 bits (compress-gate logits)
    valid: np.ndarray             # [sum T] uint8
    req_start: np.ndarray         # [B + 1] int32
    ape: np.ndarray               # [kpool, 128] float32
    ln_w: np.ndarray              # [128] bf16 bits
    ln_b: np.ndarray              # [128] bf16 bits
    q_mla: np.ndarray             # [Q, hm, 512] bf16 bits
    kv: np.ndarray                # [sum T, 512] bf16 bits
    eps: float = 1e-5
    sm_scale: float = float(1.0 / np.sqrt(KV_LORA))
    notes: Dict[str, str] = field(default_factory=dict)

    @property
    def B(self) -> int:
        return len(self.lengths)

    @property
    def Q(self) -> int:
        return int(self.q_req.shape[0])

    @property
    def M(self) -> int:
        return int(self.hidden.shape[0])

    @property
    def total_tokens(self) -> int:
        return int(self.req_start[-1])

    @property
    def out_width(self) -> int:
        return self.select_k * self.kpool


def _rng(seed: int, stream: int) -> np.random.Generator:
    # One independent stream per tensor so that adding a tensor never shifts others.
    return np.random.default_rng([seed, stream])


def _normal_bf16(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return f32_to_bf16_bits(x)


def build(name: str, *, lengths: List[int], pads: List[int], kpool: int, max_pools: int,
          select_k: int, hm: int, q_req: List[int], q_pos: List[int], seed: int = 0,
          gate_sigma: float = 1.0, holes: Optional[List[int]] = None) -> Workload:
    """Draw every input array for the given geometry.

    ``holes`` lists absolute token rows whose validity byte is cleared on top of
    the left padding (used by edge-case tests).
    """
    lengths = [int(t) for t in lengths]
    pads = [int(p) for p in pads]
    assert len(lengths) == len(pads)
    req_start = np.zeros(len(lengths) + 1, dtype=np.int32)
    req_start[1:] = np.cumsum(lengths, dtype=np.int64).astype(np.int32)
    total = int(req_start[-1])
    n_q = len(q_req)

    valid = np.ones(total, dtype=np.uint8)
    for b, p in enumerate(pads):
        valid[req_start[b]:req_start[b] + min(p, lengths[b])] = 0
    if holes:
        valid[np.asarray(holes, dtype=np.int64)] = 0

    hidden = _rng(seed, 1).standard_normal((n_q, HIDDEN), dtype=np.float32)
    w_gate = _rng(seed, 2).standard_normal((HIDDEN, INDEX_HEADS), dtype=np.float32)
    w_gate *= np.float32(1.0 / 64.0)
    q_idx = _normal_bf16(_rng(seed, 3), (n_q, INDEX_HEADS, INDEX_DIM), 1.0)
    k = _normal_bf16(_rng(seed, 4), (total, INDEX_DIM), 1.0)
    gate = _normal_bf16(_rng(seed, 5), (total, INDEX_DIM), gate_sigma)
    ape = _rng(seed, 6).standard_normal((kpool, INDEX_DIM), dtype=np.float32) * np.float32(0.02)
    r7 = _rng(seed, 7)
    ln_w = f32_to_bf16_bits(1.0 + 0.02 * r7.standard_normal(INDEX_DIM, dtype=np.float32))
    ln_b = f32_to_bf16_bits(0.02 * r7.standard_normal(INDEX_DIM, dtype=np.float32))
    q_mla = _normal_bf16(_rng(seed, 8), (n_q, hm, KV_LORA), 1.0)
    kv = _normal_bf16(_rng(seed, 9), (total, KV_LORA), 1.0)

    return Workload(
        name=name, seed=seed, kpool=kpool, max_pools=max_pools, select_k=select_k, hm=hm,
        lengths=lengths, pads=pads,
        q_req=np.asarray(q_req, dtype=np.int32), q_pos=np.asarray(q_pos, dtype=np.int32),
        hidden=hidden, w_gate=w_gate, q_idx=q_idx, k=k, gate=gate, valid=valid,
        req_start=req_start, ape=ape.astype(np.float32), ln_w=ln_w, ln_b=ln_b,
        q_mla=q_mla, kv=kv)


def _decode_queries(lengths: List[int]):
    # Decode: one query per request, at the request's last cached token.
    return list(range(len(lengths))), [t - 1 for t in lengths]


def tiny(seed: int = 0) -> Workload:
    """1 query over 512 tokens, first 16 invalid; kpool 4, 16 pools selected, MLA 16 heads."""
    lengths, pads = [512], [16]
    qr, qp = _decode_queries(lengths)
    return build("tiny decode 1x512 (pad 16) kpool4 sel16 hm16", lengths=lengths, pads=pads,
                 kpool=4, max_pools=128, select_k=16, hm=16, q_req=qr, q_pos=qp, seed=seed)


def batched(seed: int = 0, n_req: int = 16, ctx: int = 8192) -> Workload:
    """16 requests x 8192 tokens, left pad U{0..64}; kpool 4 (2048 pools), 512 pools selected."""
    pads = [int(p) for p in _rng(seed, 100).integers(0, 65, size=n_req)]
    lengths = [ctx] * n_req
    qr, qp = _decode_queries(lengths)
    return build(f"batched decode {n_req}x{ctx} (pad U0-64) kpool4 sel512 hm64", lengths=lengths,
                 pads=pads, kpool=4, max_pools=(ctx + 3) // 4, select_k=512, hm=64,
                 q_req=qr, q_pos=qp, seed=seed)


def ragged(seed: int = 0, n_req: int = 64, lo_pools: int = 128, hi_pools: int = 4095) -> Workload:
    """64 requests, T uniform in 1024-32768 with a 1..7-token trailing partial pool; kpool 8."""
    r = _rng(seed, 101)
    n = r.integers(lo_pools, hi_pools + 1, size=n_req)
    tail = r.integers(1, 8, size=n_req)
    lengths = [int(8 * a + t) for a, t in zip(n, tail)]
    qr, qp = _decode_queries(lengths)
    max_pools = (hi_pools * 8 + 7 + 7) // 8
    return build(f"ragged decode {n_req}xU[1024,32768] kpool8 sel256 hm64", lengths=lengths,
                 pads=[0] * n_req, kpool=8, max_pools=max_pools, select_k=256, hm=64,
                 q_req=qr, q_pos=qp, seed=seed)


def long_ctx(seed: int = 0, n_req: int = 4, ctx: int = 131072) -> Workload:
    """4 requests x 131072 tokens; kpool 4 (32768 pools), 512 selected; gate logits N(0,2)."""
    lengths = [ctx] * n_req
    qr, qp = _decode_queries(lengths)
    return build(f"long-context decode {n_req}x{ctx} kpool4 sel512 hm64", lengths=lengths,
                 pads=[0] * n_req, kpool=4, max_pools=(ctx + 3) // 4, select_k=512, hm=64,
                 q_req=qr, q_pos=qp, seed=seed, gate_sigma=2.0)


def prefill(seed: int = 0, ctx: int = 16384, n_q: int = 2048) -> Workload:
    """One request, 2048 queries at positions ctx-2048..ctx-1 with causal candidate pools."""
    qp = list(range(ctx - n_q, ctx))
    return build(f"chunked prefill {n_q}q over {ctx} kpool4 sel512 hm64", lengths=[ctx], pads=[0],
                 kpool=4, max_pools=(ctx + 3) // 4, select_k=512, hm=64,
                 q_req=[0] * n_q, q_pos=qp, seed=seed)


CONFIGS = {
    "tiny": tiny,
    "batched": batched,
    "ragged": ragged,
    "long": long_ctx,
    "prefill": prefill,
}


def make(name: str, seed: int = 0, **kw) -> Workload:
    return CONFIGS[name](seed=seed, **kw)
