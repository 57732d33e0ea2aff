"""ctypes binding of libdsa.so (include/dsa.h), one Python function per C entry point.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Pointer arguments accept a torch tensor (its data_ptr()), an int
address or None; ``stream`` accepts a torch.cuda.Stream, an int handle or None
(torch's current stream). A non-OK status raises DsaError. There is no
fallback: importing this module fails loudly when libdsa.so is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_ALIGNMENT = 3
DSA_ERR_WORKSPACE = 4
DSA_ERR_CUDA = 5

# Every symbol include/dsa.h declares.
EXPORTS = (
    "dsa_status_string", "dsa_abi_version", "dsa_device_status", "dsa_selftest_bounded_wait",
    "dsa_head_gate", "dsa_head_gate_supported",
    "dsa_kpool_compress", "dsa_indexer_store", "dsa_kpool_compress_tokens",
    "dsa_index_scores", "dsa_topk_expand", "dsa_topk_expand_tail", "dsa_indexer_select",
    "dsa_sparse_mla_workspace_size", "dsa_sparse_mla_launch_count", "dsa_sparse_mla_decode",
    "dsa_sparse_mla_decode_noalloc", "dsa_sparse_mla_decode_paged",
    "dsa_sparse_mla_decode_paged_fp8", "dsa_noalloc_scratch_bytes",
)


class DsaError(RuntimeError):
    def __init__(self, fn: str, status: int, name: str):
        super().__init__(f"{fn} failed: {name} ({status})")
        self.status = status
        self.name = name


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libdsa.so not found at {LIB_PATH}; build it with "
            "`python -m sparse_attention_indexer_head_b200.build` (no fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    I64 = ctypes.c_int64
    sig = {
        "dsa_status_string": ([I], ctypes.c_char_p),
        "dsa_abi_version": ([], I),
        "dsa_device_status": ([ctypes.POINTER(I), I], I),
        "dsa_selftest_bounded_wait": ([P, P], I),
        "dsa_head_gate": ([P, P, P, I, I, I, P], I),
        "dsa_head_gate_supported": ([I, I, I], I),
        "dsa_kpool_compress": ([P, P, P, P, I, I, I, I, P, P, P, F, P, P, P, P, P], I),
        "dsa_indexer_store": ([P, P, P, P, P, I, I, P, I, P, P, P, P], I),
        "dsa_kpool_compress_tokens": ([P, P, P, P, I, I, I, I, P, P, P, F, P, P, P, P, P, P, P],
                                      I),
        "dsa_index_scores": ([P, P, P, P, I, I, I, P, P, P, I, I, I, P, P, P], I),
        "dsa_topk_expand": ([P, P, P, P, I, I, I, I, I, P, P, P], I),
        "dsa_topk_expand_tail": ([P, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P], I),
        "dsa_indexer_select": ([P, P, I, P, P, P, I, I, I, P, P, P, P, I, I, I, I, P, P, P, P, P, P],
                               I),
        "dsa_sparse_mla_workspace_size": ([I, I, I], Z),
        "dsa_sparse_mla_launch_count": ([I, I, I], I),
        "dsa_sparse_mla_decode": ([P, P, I64, P, P, P, I, I, I, I, I, I, F, P, P, P, Z, P], I),
        "dsa_sparse_mla_decode_noalloc": ([P, P, I64, P, P, P, I, I, I, I, I, I, F, P, P, P], I),
        "dsa_noalloc_scratch_bytes": ([], Z),
        "dsa_sparse_mla_decode_paged": ([P, P, I64, P, I, I, P, P, P, I, I, I, I, I, I, F, P, P, P,
                                         Z, P], I),
        "dsa_sparse_mla_decode_paged_fp8": ([P, P, F, I64, P, I, I, P, P, P, I, I, I, I, I, I, F, P,
                                             P, P, Z, P], I),
    }
    for name, (argtypes, restype) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = argtypes
        fn.restype = restype
    return L


lib = _load()
# Size of the library's own scratch for dsa_sparse_mla_decode_noalloc, as built.
DSA_NOALLOC_SCRATCH_BYTES = int(lib.dsa_noalloc_scratch_bytes())


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != DSA_OK:
        raise DsaError(fn, status, dsa_status_string(status))


def dsa_status_string(status: int) -> str:
    return lib.dsa_status_string(int(status)).decode()


def dsa_abi_version() -> int:
    return int(lib.dsa_abi_version())


def dsa_device_status(reset: bool = True) -> int:
    v = ctypes.c_int(0)
    _check("dsa_device_status", lib.dsa_device_status(ctypes.byref(v), int(reset)))
    return v.value


def dsa_selftest_bounded_wait(result, stream=None) -> None:
    _check("dsa_selftest_bounded_wait", lib.dsa_selftest_bounded_wait(_ptr(result), _stream(stream)))


def dsa_head_gate_supported(M: int, K: int, N: int) -> bool:
    return int(lib.dsa_head_gate_supported(M, K, N)) == DSA_OK


def dsa_head_gate(hidden, w, out, M: int, K: int, N: int, stream=None) -> None:
    _check("dsa_head_gate", lib.dsa_head_gate(_ptr(hidden), _ptr(w), _ptr(out), M, K, N,
                                              _stream(stream)))


def dsa_kpool_compress(k, gate, tok_valid, req_start, B: int, D: int, kpool: int, max_pools: int,
                       ape, ln_w, ln_b, eps: float, pool_keys, pool_idx, pool_valid, first_valid,
                       stream=None) -> None:
    _check("dsa_kpool_compress", lib.dsa_kpool_compress(
        _ptr(k), _ptr(gate), _ptr(tok_valid), _ptr(req_start), B, D, kpool, max_pools, _ptr(ape),
        _ptr(ln_w), _ptr(ln_b), float(eps), _ptr(pool_keys), _ptr(pool_idx), _ptr(pool_valid),
        _ptr(first_valid), _stream(stream)))


def dsa_indexer_store(k_new, gate_new, valid_new, tok_req, tok_pos, n: int, D: int, req_start,
                      B: int, k, gate, tok_valid, stream=None) -> None:
    _check("dsa_indexer_store", lib.dsa_indexer_store(
        _ptr(k_new), _ptr(gate_new), _ptr(valid_new), _ptr(tok_req), _ptr(tok_pos), n, D,
        _ptr(req_start), B, _ptr(k), _ptr(gate), _ptr(tok_valid), _stream(stream)))


def dsa_kpool_compress_tokens(k, gate, tok_valid, req_start, B: int, D: int, kpool: int,
                              max_pools: int, ape, ln_w, ln_b, eps: float, tok_begin, tok_end,
                              pool_keys, pool_idx, pool_valid, first_valid, stream=None) -> None:
    _check("dsa_kpool_compress_tokens", lib.dsa_kpool_compress_tokens(
        _ptr(k), _ptr(gate), _ptr(tok_valid), _ptr(req_start), B, D, kpool, max_pools, _ptr(ape),
        _ptr(ln_w), _ptr(ln_b), float(eps), _ptr(tok_begin), _ptr(tok_end), _ptr(pool_keys),
        _ptr(pool_idx), _ptr(pool_valid), _ptr(first_valid), _stream(stream)))


def dsa_index_scores(q_idx, gate_w, q_req, q_pos, Q: int, H: int, D: int, pool_keys, pool_valid,
                     first_valid, B: int, kpool: int, max_pools: int, scores, cand,
                     stream=None) -> None:
    _check("dsa_index_scores", lib.dsa_index_scores(
        _ptr(q_idx), _ptr(gate_w), _ptr(q_req), _ptr(q_pos), Q, H, D, _ptr(pool_keys),
        _ptr(pool_valid), _ptr(first_valid), B, kpool, max_pools, _ptr(scores), _ptr(cand),
        _stream(stream)))


def dsa_topk_expand(scores, cand, pool_idx, q_req, Q: int, B: int, max_pools: int, kpool: int,
                    select_k: int, top_pools, token_ids, stream=None) -> None:
    _check("dsa_topk_expand", lib.dsa_topk_expand(
        _ptr(scores), _ptr(cand), _ptr(pool_idx), _ptr(q_req), Q, B, max_pools, kpool, select_k,
        _ptr(top_pools), _ptr(token_ids), _stream(stream)))


def dsa_topk_expand_tail(scores, cand, pool_idx, q_req, q_pos, first_valid, tok_valid, req_start,
                         Q: int, B: int, max_pools: int, kpool: int, select_k: int, top_pools,
                         token_ids, stream=None) -> None:
    _check("dsa_topk_expand_tail", lib.dsa_topk_expand_tail(
        _ptr(scores), _ptr(cand), _ptr(pool_idx), _ptr(q_req), _ptr(q_pos), _ptr(first_valid),
        _ptr(tok_valid), _ptr(req_start), Q, B, max_pools, kpool, select_k, _ptr(top_pools),
        _ptr(token_ids), _stream(stream)))


def dsa_indexer_select(hidden, w, K: int, q_idx, q_req, q_pos, Q: int, H: int, D: int, pool_keys,
                       pool_valid, first_valid, pool_idx, B: int, kpool: int, max_pools: int,
                       select_k: int, gate_w, scores, cand, top_pools, token_ids,
                       stream=None) -> None:
    _check("dsa_indexer_select", lib.dsa_indexer_select(
        _ptr(hidden), _ptr(w), K, _ptr(q_idx), _ptr(q_req), _ptr(q_pos), Q, H, D, _ptr(pool_keys),
        _ptr(pool_valid), _ptr(first_valid), _ptr(pool_idx), B, kpool, max_pools, select_k,
        _ptr(gate_w), _ptr(scores), _ptr(cand), _ptr(top_pools), _ptr(token_ids), _stream(stream)))


def dsa_sparse_mla_workspace_size(Q: int, Hm: int, W: int) -> int:
    return int(lib.dsa_sparse_mla_workspace_size(Q, Hm, W))


def dsa_sparse_mla_launch_count(Q: int, Hm: int, W: int) -> int:
    return int(lib.dsa_sparse_mla_launch_count(Q, Hm, W))


def dsa_sparse_mla_decode(q, kv, kv_rows: int, req_start, q_req, token_ids, Q: int, B: int,
                          Hm: int, W: int, kv_lora: int, rope_dim: int, sm_scale: float, out, lse,
                          workspace, workspace_bytes: int, stream=None) -> None:
    _check("dsa_sparse_mla_decode", lib.dsa_sparse_mla_decode(
        _ptr(q), _ptr(kv), int(kv_rows), _ptr(req_start), _ptr(q_req), _ptr(token_ids), Q, B, Hm, W, kv_lora,
        rope_dim, float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace), int(workspace_bytes),
        _stream(stream)))


def dsa_sparse_mla_decode_noalloc(q, kv, kv_rows: int, req_start, q_req, token_ids, Q: int,
                                  B: int, Hm: int, W: int, kv_lora: int, rope_dim: int,
                                  sm_scale: float, out, lse, stream=None) -> None:
    """dsa_sparse_mla_decode for callers that cannot allocate: the split-KV scratch is the
    library's own static device area (see include/dsa.h)."""
    _check("dsa_sparse_mla_decode_noalloc", lib.dsa_sparse_mla_decode_noalloc(
        _ptr(q), _ptr(kv), int(kv_rows), _ptr(req_start), _ptr(q_req), _ptr(token_ids), Q, B, Hm, W, kv_lora,
        rope_dim, float(sm_scale), _ptr(out), _ptr(lse), _stream(stream)))


def dsa_sparse_mla_decode_paged(q, kv, kv_rows: int, block_table, max_blocks: int, page_size: int,
                                seq_len, q_req, token_ids, Q: int, B: int, Hm: int, W: int,
                                kv_lora: int, rope_dim: int, sm_scale: float, out, lse, workspace,
                                workspace_bytes: int, stream=None) -> None:
    _check("dsa_sparse_mla_decode_paged", lib.dsa_sparse_mla_decode_paged(
        _ptr(q), _ptr(kv), kv_rows, _ptr(block_table), max_blocks, page_size, _ptr(seq_len),
        _ptr(q_req), _ptr(token_ids), Q, B, Hm, W, kv_lora, rope_dim, float(sm_scale), _ptr(out),
        _ptr(lse), _ptr(workspace), workspace_bytes, _stream(stream)))


def dsa_sparse_mla_decode_paged_fp8(q, kv8, kv_scale: float, kv_rows: int, block_table,
                                    max_blocks: int, page_size: int, seq_len, q_req, token_ids,
                                    Q: int, B: int, Hm: int, W: int, kv_lora: int, rope_dim: int,
                                    sm_scale: float, out, lse, workspace, workspace_bytes: int,
                                    stream=None) -> None:
    _check("dsa_sparse_mla_decode_paged_fp8", lib.dsa_sparse_mla_decode_paged_fp8(
        _ptr(q), _ptr(kv8), float(kv_scale), kv_rows, _ptr(block_table), max_blocks, page_size,
        _ptr(seq_len), _ptr(q_req), _ptr(token_ids), Q, B, Hm, W, kv_lora, rope_dim,
        float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace_bytes, _stream(stream)))
