"""One DSA decode/prefill step on the GPU: device buffers plus the C-ABI calls.

PyTorch is used for device memory, pinned host memory and streams only; every
stage runs in libdsa.so:
  dsa_kpool_compress -> dsa_head_gate -> dsa_index_scores -> dsa_topk_expand
  -> dsa_sparse_mla_decode,
or, with the fused indexer, dsa_kpool_compress -> dsa_indexer_select (gate,
scores, top-k and expansion in one launch) -> dsa_sparse_mla_decode.
Cache-side tensors (k, gate logits, validity, latent kv, request offsets and
the layer weights) are device-resident state; query-side tensors (hidden,
indexer queries, MLA queries, query request/position) are the per-step inputs.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B
from .workloads import INDEX_DIM, INDEX_HEADS, KV_LORA, Workload

QUERY_INPUTS = ("hidden", "q_idx", "q_mla", "q_req", "q_pos")
INDEXER_MAX_POOLS = 32768          # dsa_indexer_select's pool limit
AUTO_FUSED_MAX_QUERIES = 256       # "auto": the fused indexer up to this many queries


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def host_tensors(wl: Workload) -> Dict[str, torch.Tensor]:
    """CPU torch views of a workload's arrays (bf16 bit patterns as torch.bfloat16)."""
    return {
        "hidden": torch.from_numpy(wl.hidden),
        "w_gate": torch.from_numpy(wl.w_gate),
        "q_idx": _bf16(wl.q_idx),
        "k": _bf16(wl.k),
        "gate": _bf16(wl.gate),
        "valid": torch.from_numpy(wl.valid),
        "req_start": torch.from_numpy(wl.req_start),
        "ape": torch.from_numpy(wl.ape),
        "ln_w": _bf16(wl.ln_w),
        "ln_b": _bf16(wl.ln_b),
        "q_mla": _bf16(wl.q_mla),
        "kv": _bf16(wl.kv),
        "q_req": torch.from_numpy(wl.q_req),
        "q_pos": torch.from_numpy(wl.q_pos),
    }


@dataclass
class Geometry:
    B: int
    Q: int
    kpool: int
    max_pools: int
    select_k: int
    hm: int
    eps: float
    sm_scale: float
    tail: int = 0           # always_select_tail: kpool - 1 extra slots per index row

    @property
    def W(self) -> int:
        return self.select_k * self.kpool + self.tail


class DecodeStep:
    """Device buffers of one step; ``run()`` enqueues the five calls on a stream."""

    def __init__(self, wl: Workload, device: str = "cuda", inputs: Optional[Dict] = None,
                 always_select_tail: bool = False, fused_indexer: bool = False):
        self.device = torch.device(device)
        # fused_indexer: gate, scores, top-k and expansion in one dsa_indexer_select
        # call (not with always_select_tail, whose tail slots only dsa_topk_expand_tail
        # writes, nor above its pool limit). "auto" takes it for decode-sized batches:
        # its cluster of 8 CTAs a query recomputes the gate and re-reads the request's
        # pooled keys per query, which the separate calls amortise over many queries.
        if fused_indexer == "auto":
            fused_indexer = wl.Q <= AUTO_FUSED_MAX_QUERIES
        self.fused = (bool(fused_indexer) and not always_select_tail
                      and wl.max_pools <= INDEXER_MAX_POOLS)
        self.g = Geometry(wl.B, wl.Q, wl.kpool, wl.max_pools, wl.select_k, wl.hm, wl.eps,
                          wl.sm_scale, wl.kpool - 1 if always_select_tail else 0)
        src = host_tensors(wl) if inputs is None else inputs
        self.t = {k: v.to(self.device) for k, v in src.items()}
        g, dev = self.g, self.device
        self.gate_w = torch.empty(g.Q, INDEX_HEADS, dtype=torch.float32, device=dev)
        self.pool_keys = torch.zeros(g.B, g.max_pools, INDEX_DIM, dtype=torch.bfloat16, device=dev)
        self.pool_idx = torch.empty(g.B, g.max_pools, g.kpool, dtype=torch.int32, device=dev)
        self.pool_valid = torch.empty(g.B, g.max_pools, dtype=torch.uint8, device=dev)
        self.first_valid = torch.empty(g.B, dtype=torch.int32, device=dev)
        self.scores = torch.empty(g.Q, g.max_pools, dtype=torch.float32, device=dev)
        self.cand = torch.empty(g.Q, g.max_pools, dtype=torch.uint8, device=dev)
        self.top_pools = torch.empty(g.Q, g.select_k, dtype=torch.int32, device=dev)
        self.token_ids = torch.empty(g.Q, g.W, dtype=torch.int32, device=dev)
        self.out = torch.empty(g.Q, g.hm, KV_LORA, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(g.Q, g.hm, dtype=torch.float32, device=dev)
        ws = B.dsa_sparse_mla_workspace_size(g.Q, g.hm, g.W)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)

    # -- the five stages ---------------------------------------------------------------
    def head_gate(self, stream=None):
        g, t = self.g, self.t
        B.dsa_head_gate(t["hidden"], t["w_gate"], self.gate_w, g.Q, t["hidden"].shape[1],
                        INDEX_HEADS, stream)

    def kpool_compress(self, stream=None):
        g, t = self.g, self.t
        B.dsa_kpool_compress(t["k"], t["gate"], t["valid"], t["req_start"], g.B, INDEX_DIM,
                             g.kpool, g.max_pools, t["ape"], t["ln_w"], t["ln_b"], g.eps,
                             self.pool_keys, self.pool_idx, self.pool_valid, self.first_valid,
                             stream)

    def index_scores(self, stream=None):
        g, t = self.g, self.t
        B.dsa_index_scores(t["q_idx"], self.gate_w, t["q_req"], t["q_pos"], g.Q, INDEX_HEADS,
                           INDEX_DIM, self.pool_keys, self.pool_valid, self.first_valid, g.B,
                           g.kpool, g.max_pools, self.scores, self.cand, stream)

    def topk_expand(self, stream=None):
        g, t = self.g, self.t
        if g.tail:
            B.dsa_topk_expand_tail(self.scores, self.cand, self.pool_idx, t["q_req"], t["q_pos"],
                                   self.first_valid, t["valid"], t["req_start"], g.Q, g.B,
                                   g.max_pools, g.kpool, g.select_k, self.top_pools,
                                   self.token_ids, stream)
        else:
            B.dsa_topk_expand(self.scores, self.cand, self.pool_idx, t["q_req"], g.Q, g.B,
                              g.max_pools, g.kpool, g.select_k, self.top_pools, self.token_ids,
                              stream)

    def sparse_mla(self, stream=None):
        g, t = self.g, self.t
        B.dsa_sparse_mla_decode(t["q_mla"], t["kv"], t["kv"].shape[0], t["req_start"], t["q_req"],
                                self.token_ids,
                                g.Q, g.B, g.hm, g.W, KV_LORA, 0, g.sm_scale, self.out, self.lse,
                                self.ws, self.ws.numel(), stream)

    def indexer(self, stream=None):
        """a1 + a4 + a5 + a6 in one launch (dsa_indexer_select)."""
        g, t = self.g, self.t
        B.dsa_indexer_select(t["hidden"], t["w_gate"], t["hidden"].shape[1], t["q_idx"], t["q_req"],
                             t["q_pos"], g.Q, INDEX_HEADS, INDEX_DIM, self.pool_keys,
                             self.pool_valid, self.first_valid, self.pool_idx, g.B, g.kpool,
                             g.max_pools, g.select_k, self.gate_w, self.scores, self.cand,
                             self.top_pools, self.token_ids, stream)

    def stages(self):
        """Names of the stage methods run() calls, in order."""
        if self.fused:
            return ["kpool_compress", "indexer", "sparse_mla"]
        # compress first: the small head-gate grid then overlaps compress's tail
        # (every kernel is launched with programmatic dependent launch).
        return ["kpool_compress", "head_gate", "index_scores", "topk_expand", "sparse_mla"]

    def run(self, stream=None):
        for name in self.stages():
            getattr(self, name)(stream)

    # -- incremental decode: the step's new token rows update the pooled-key cache -------
    def stage_new_tokens(self, k_new=None, gate_new=None, valid_new=None, tok_req=None,
                         tok_pos=None):
        """Device buffers of a step's new indexer rows and the token ranges they change.

        Default: one new token per request, its last row (position T_b - 1), with
        the k and gate values the cache already holds there, so a step that
        stores it leaves the cache as it was and its outputs can be compared
        with the full step's. Requests with no rows get none.
        """
        g, t, dev = self.g, self.t, self.device
        rs = t["req_start"].to("cpu").numpy().astype(np.int64)
        lengths = rs[1:] - rs[:-1]
        if tok_req is None:
            have = np.nonzero(lengths > 0)[0]
            tok_req = have.astype(np.int32)
            tok_pos = (lengths[have] - 1).astype(np.int32)
            rows = torch.from_numpy(rs[have] + tok_pos).to(dev)
            k_new = t["k"].index_select(0, rows)
            gate_new = t["gate"].index_select(0, rows)
            valid_new = t["valid"].index_select(0, rows)
        tok_req = np.asarray(tok_req, np.int32)
        tok_pos = np.asarray(tok_pos, np.int32)
        begin = np.full(g.B, 0, np.int32)
        end = np.full(g.B, 0, np.int32)
        for b in range(g.B):                   # the smallest range holding b's new rows
            mine = tok_pos[tok_req == b]
            if mine.size:
                begin[b], end[b] = mine.min(), mine.max() + 1
        self.new = {
            "k": torch.as_tensor(k_new).to(dev), "gate": torch.as_tensor(gate_new).to(dev),
            "valid": None if valid_new is None else torch.as_tensor(valid_new).to(dev),
            "tok_req": torch.from_numpy(tok_req).to(dev), "tok_pos": torch.from_numpy(tok_pos).to(dev),
            "n": int(tok_req.shape[0]),
            "tok_begin": torch.from_numpy(begin).to(dev), "tok_end": torch.from_numpy(end).to(dev),
        }

    def indexer_store(self, stream=None):
        g, t, n = self.g, self.t, self.new
        B.dsa_indexer_store(n["k"], n["gate"], n["valid"], n["tok_req"], n["tok_pos"], n["n"],
                            INDEX_DIM, t["req_start"], g.B, t["k"], t["gate"], t["valid"], stream)

    def kpool_compress_tokens(self, stream=None):
        g, t, n = self.g, self.t, self.new
        B.dsa_kpool_compress_tokens(t["k"], t["gate"], t["valid"], t["req_start"], g.B, INDEX_DIM,
                                    g.kpool, g.max_pools, t["ape"], t["ln_w"], t["ln_b"], g.eps,
                                    n["tok_begin"], n["tok_end"], self.pool_keys, self.pool_idx,
                                    self.pool_valid, self.first_valid, stream)

    def run_incremental(self, stream=None):
        """A decode step that stores the new rows and recomputes only their pools.

        The pooled-key outputs must already hold the compress result of the
        cache before the new rows (run() or kpool_compress() once).
        """
        self.indexer_store(stream)
        self.kpool_compress_tokens(stream)
        for name in self.stages()[1:]:
            getattr(self, name)(stream)

    def kernels_per_step(self) -> int:
        """Launches of run(): compress, then gate, scores and topk+expand (or the one fused
        indexer), and the MLA's one or two kernels (split kernel, plus the combine when
        splits merge in the workspace)."""
        g = self.g
        return len(self.stages()) - 1 + B.dsa_sparse_mla_launch_count(g.Q, g.hm, g.W)

    def kernels_per_step_incremental(self) -> int:
        """Launches of run_incremental(): store (when there are new rows), token-range
        compress, the indexer stage(s) and the MLA's kernels."""
        return (1 if self.new["n"] > 0 else 0) + self.kernels_per_step()

    def outputs_numpy(self) -> Dict[str, np.ndarray]:
        def u16(x):
            return x.view(torch.int16).cpu().numpy().view(np.uint16)
        return {
            "gate_w": self.gate_w.cpu().numpy(),
            "pool_keys": u16(self.pool_keys),
            "pool_idx": self.pool_idx.cpu().numpy(),
            "pool_valid": self.pool_valid.cpu().numpy(),
            "first_valid": self.first_valid.cpu().numpy(),
            "scores": self.scores.cpu().numpy(),
            "cand": self.cand.cpu().numpy(),
            "top_pools": self.top_pools.cpu().numpy(),
            "token_ids": self.token_ids.cpu().numpy(),
            "out": u16(self.out),
            "lse": self.lse.cpu().numpy(),
        }


class StreamedDecode:
    """Decode steps served from and to pinned host memory.

    Each slot owns a pinned host input buffer (the query inputs packed, see
    `write_inputs`), device buffers and a pinned host output buffer, and a CUDA
    graph that copies the inputs host -> device, runs the five calls and copies
    the output device -> host, on the slot's own stream. Steps rotate over the
    slots, so consecutive steps run on different streams and overlap on the
    GPU (their copies and kernels interleave). Step i uses slot i % slots: its
    inputs must be in that slot's buffer when it is submitted, and the buffer
    may be refilled for step i + slots once result(i) has returned.
    """

    def __init__(self, wl: Workload, device: str = "cuda", slots: int = 2,
                 inputs: Optional[Dict] = None, fused_indexer: bool = False):
        self.device = torch.device(device)
        self.steps = [DecodeStep(wl, device=device, inputs=inputs, fused_indexer=fused_indexer)
                      for _ in range(slots)]
        # A slot's query inputs live in one device buffer: one copy per step.
        self.layout, nbytes = {}, 0
        for name in QUERY_INPUTS:
            t = self.steps[0].t[name]
            nbytes = (nbytes + 255) // 256 * 256
            self.layout[name] = (nbytes, t.dtype, tuple(t.shape))
            nbytes += t.numel() * t.element_size()
        self.nbytes = nbytes
        self.dev_in, self.in_host, self.out_host, self.streams = [], [], [], []
        for st in self.steps:
            buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            host = torch.zeros(nbytes, dtype=torch.uint8).pin_memory()
            for name, (off, dtype, shape) in self.layout.items():
                view = self._view(buf, off, dtype, shape)
                view.copy_(st.t[name])
                self._view(host, off, dtype, shape).copy_(st.t[name].cpu())
                st.t[name] = view
            self.dev_in.append(buf)
            self.in_host.append(host)
            self.out_host.append(torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory())
            self.streams.append(torch.cuda.Stream(device=self.device))
        self.graphs = []
        for k, st in enumerate(self.steps):
            with torch.cuda.stream(self.streams[k]):
                st.run()                                  # sets kernel attributes eagerly
            self.streams[k].synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.streams[k]):
                self.dev_in[k].copy_(self.in_host[k], non_blocking=True)
                st.run()
                self.out_host[k].copy_(st.out, non_blocking=True)
            self.graphs.append(g)
        torch.cuda.synchronize(self.device)
        self.done = [torch.cuda.Event() for _ in self.steps]
        self.submitted = 0

    @staticmethod
    def _view(buf: torch.Tensor, off: int, dtype, shape) -> torch.Tensor:
        n = 1
        for d in shape:
            n *= d
        size = n * torch.empty((), dtype=dtype).element_size()
        return buf[off:off + size].view(dtype).view(shape)

    def slot(self, i: int) -> int:
        return i % len(self.steps)

    def write_inputs(self, i: int, host_inputs: Dict[str, torch.Tensor]) -> None:
        """Pack step i's query inputs (names of QUERY_INPUTS) into its slot's buffer."""
        buf = self.in_host[self.slot(i)]
        for name, (off, dtype, shape) in self.layout.items():
            self._view(buf, off, dtype, shape).copy_(host_inputs[name])

    def submit(self) -> int:
        """Enqueue the next step on its slot's stream; returns its index."""
        i = self.submitted
        k = self.slot(i)
        with torch.cuda.stream(self.streams[k]):
            self.graphs[k].replay()
            self.done[k].record(self.streams[k])
        self.submitted += 1
        return i

    def result(self, i: int) -> torch.Tensor:
        """Step i's output [Q, Hm, 512] bf16 on the host (step i must be among the
        last `slots` submitted)."""
        if not (self.submitted - len(self.steps) <= i < self.submitted):
            raise ValueError("step is not among the slots in flight")
        self.done[self.slot(i)].synchronize()
        return self.out_host[self.slot(i)]

    def kernels_per_step(self) -> int:
        return self.steps[0].kernels_per_step()
