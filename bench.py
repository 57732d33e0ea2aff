#!/usr/bin/env python3
"""Benchmark of the DSA decode hot path on B200 (one JSON line per workload on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--config tiny|batched|ragged|long|prefill|all]

A step is one pass of the whole path -- head gate, kpool_compress (+k_norm),
index_scores, top-k + expand, sparse NoPE MLA -- over one batch of a seeded
synthetic workload. The default workload (the headline line) is the batched
decode: 16 requests x 8192 cached tokens (left pad U{0..64}), kpool 4 (2048
pools), 512 pools (2048 tokens) selected per query, 64 MLA heads over a
512-wide NoPE latent. --config names another workload (tiny 1x512, ragged
64 x U[1024,32768], long-context 4 x 131072, chunked prefill of 2048 queries
over 16384 tokens) or "all", which prints one line for each.

Timing: CUDA graphs of the step's kernel launches, replayed over device-resident
input sets that together exceed the 126 MB L2 (three for the batched decode,
as many as that takes for the small tiny workload), so no step reads another
step's inputs from L2; CUDA events on the launching stream with a barrier and a
synchronize on both sides; the max over ranks. Under torchrun each rank runs
its own batch (weak scaling; the path has no exchange step, so there is no
collective on the data path -- replicas only).

--impl reference times the CPU oracle (the test oracle, plain C, binary64) on
the host cores, on a bounded sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode queries/sec and achieved HBM GB/s (% of B200 peak) for DSA indexer+sparse MLA"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------- bytes
def algorithmic_bytes(wl) -> dict:
    """Bytes each stage must move at least once (inputs read once, outputs written once)."""
    D, H, L, kp, P = 128, 16, 512, wl.kpool, wl.max_pools
    T = np.diff(wl.req_start).astype(np.int64)
    f = np.array([next((i for i in range(t) if wl.valid[s + i]), t)
                  for s, t in zip(wl.req_start[:-1], T)], dtype=np.int64)
    n_span = np.minimum(P, (T - f) // kp)
    Q = wl.Q
    gate = 4 * (wl.M * wl.hidden.shape[1] + wl.hidden.shape[1] * H + H * wl.M)
    compress = int((n_span * kp * (2 * D + 2 * D + 1)).sum() + (n_span * 2 * D).sum()
                   + wl.B * P * (4 * kp + 1) + 4 * wl.B + 4 * (wl.B + 1))
    # scores: each request's span keys once, per query its q/gate rows and [P] outputs
    scores = int((n_span * 2 * D).sum() + Q * (2 * H * D + 4 * H + P * (1 + 4 + 1) + 8))
    n_sel = np.minimum(wl.select_k, n_span[wl.q_req])          # pools selected (decode: all cand)
    topk = int(Q * P * 5 + (n_sel * kp * 4).sum() + Q * (4 * wl.select_k + 4 * wl.out_width + 4))
    # MLA: each request's latent rows once, the rows its queries select together; at
    # most every row of its span (prefill's 2048 queries re-read their shared rows
    # from L2), and exactly the selected rows at decode (one query a request)
    rows_b = np.zeros(wl.B, dtype=np.int64)
    np.add.at(rows_b, wl.q_req, n_sel * kp)
    rows_b = np.minimum(rows_b, n_span * kp)
    mla = int(rows_b.sum() * L * 2 + Q * (wl.hm * L * 2 * 2 + 4 * wl.out_width + 4 * wl.hm + 4))
    out = dict(head_gate=gate, kpool_compress=compress, index_scores=scores,
               topk_expand=topk, sparse_mla=mla)
    # the fused indexer moves the three stages' bytes but the ones they pass each other
    # through memory: the gate rows the scores read, the scores and flags top-k reads
    out["indexer"] = gate + scores + topk - Q * 4 * H - Q * P * 5
    return out


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, read through NVML in a
    background thread every few milliseconds (read-only queries; no setting is touched).

    The GPU is found by its PCI address from the CUDA device properties, so the
    samples are of the device the kernels run on whatever CUDA_VISIBLE_DEVICES
    holds. Start it before the warm-up; wait_first() returns once a sample exists.
    """

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.samples = []
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as N
            import torch
            pr = torch.cuda.get_device_properties(cuda_index)
            N.nvmlInit()
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self._N = N
            self._h = N.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self._max = N.nvmlDeviceGetMaxClockInfo(self._h, N.NVML_CLOCK_SM)
            self._masks = [(name, getattr(N, attr)) for name, attr in self.REASONS]
        except Exception as e:                      # no NVML: the line says so
            self.error = f"nvml unavailable: {e}"
            return
        self._period = period_s
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        N = self._N
        while not self._stop.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(self._h, N.NVML_CLOCK_SM)
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception as e:
                self.error = str(e)
                return
            self.samples.append((time.perf_counter(), sm, rs))
            time.sleep(self._period)

    def wait_first(self, timeout: float = 2.0):
        t0 = time.perf_counter()
        while self._thread and not self.samples and time.perf_counter() - t0 < timeout:
            time.sleep(0.001)

    def stop(self):
        self._stop.set()
        if self._thread:
            self._thread.join(timeout=2)

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "_max", None),
                    "reasons": [self.error or "no samples in the timed region"],
                    "samples_in_region": 0}
        reasons = sorted({name for _, _, rs in inside for name, m in self._masks if rs & m})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self._max,
                "reasons": reasons, "samples_in_region": len(inside), "source": "nvml"}


# ----------------------------------------------------------------------------- helpers
FALLBACK_TFLOPS = 1590.0            # bf16 dense, burst (the profiling recipe's fallback)


def peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, kind): MEASURED_PEAKS.json when present."""
    try:
        with open(PEAKS_FILE) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", FALLBACK_TFLOPS)), "measured"
    except (OSError, KeyError, ValueError, TypeError):
        return FALLBACK_HBM_GBS, FALLBACK_TFLOPS, "fallback"


def kernel_source_sha(kernel_file: str) -> str:
    csrc = os.path.join(ROOT, "sparse_attention_indexer_head_b200", "csrc")
    h = hashlib.sha256()
    for name in ("common.cuh", kernel_file):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# Steps in flight in the end-to-end loop (StreamedDecode slots).
E2E_SLOTS = 4
# kernel source of each stage (its DRAM traffic is valid only for that source)
STAGE_SOURCE = {"head_gate": "head_gate.cuh", "kpool_compress": "kpool_compress.cuh",
                "index_scores": "index_scores.cuh", "topk_expand": "topk_expand.cuh",
                "indexer": "indexer.cuh", "sparse_mla": "sparse_mla.cuh"}


def traffic_for(kernel: str, kernel_file: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is
    unchanged and the capture was of this workload."""
    try:
        with open(TRAFFIC_FILE) as fh:
            t = json.load(fh)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if t.get("source_sha") != kernel_source_sha(kernel_file):
        return None
    if t.get("workload_key") not in (None, workload):
        return None
    return float(t["dram_bytes_per_launch"])


def mla_flops(wl) -> float:
    """S = q K^T and O = P V over every valid selected token: 4 * Hm * 512 per (query, token)."""
    T = np.diff(wl.req_start).astype(np.int64)
    f = np.array([next((i for i in range(t) if wl.valid[s + i]), t)
                  for s, t in zip(wl.req_start[:-1], T)], dtype=np.int64)
    n_span = np.minimum(wl.max_pools, (T - f) // wl.kpool)
    b = wl.q_req
    last_ok = (wl.q_pos.astype(np.int64) - f[b] + 1) // wl.kpool      # pools ending by q_pos
    n_sel = np.minimum(wl.select_k, np.minimum(n_span[b], np.maximum(last_ok, 0)))
    return float(4 * wl.hm * 512 * (n_sel * wl.kpool).sum())


def dist_setup(backend: str = "nccl"):
    """Rank, world size and local rank from the launcher's environment; joins the
    process group when world > 1 (NCCL on GPUs; gloo serves the CPU tests)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The maximum of x over all ranks (the step time every rank reports)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(queries_per_rank: int, world: int, steps: int, seconds: float) -> float:
    """Whole-job queries/s: every rank runs its own batch each step (weak scaling),
    timed by the slowest rank."""
    return queries_per_rank * world * steps / seconds


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def input_sets(step_bytes: int, requested: int = 0) -> int:
    """Device-resident input sets the replays rotate over: together at least twice the
    L2, at least two, at most 256 (the tiny workload needs the most)."""
    if requested > 0:
        return requested
    return int(min(256, max(2, -(-2 * L2_BYTES // max(1, step_bytes)))))


# ----------------------------------------------------------------------------- oracle timing
def sample_workload(wl, queries):
    """The given queries of a workload with the requests they read, sliced out of its
    arrays (request order kept; query positions unchanged)."""
    import copy
    qs = np.asarray(queries)
    reqs = sorted(set(int(b) for b in wl.q_req[qs]))
    remap = {b: i for i, b in enumerate(reqs)}
    rows = np.concatenate([np.arange(wl.req_start[b], wl.req_start[b + 1]) for b in reqs])
    sub = copy.copy(wl)
    sub.name = wl.name + " (oracle sample)"
    sub.lengths = [wl.lengths[b] for b in reqs]
    sub.pads = [wl.pads[b] for b in reqs]
    sub.req_start = np.zeros(len(reqs) + 1, np.int32)
    sub.req_start[1:] = np.cumsum(sub.lengths)
    sub.k, sub.gate, sub.valid, sub.kv = wl.k[rows], wl.gate[rows], wl.valid[rows], wl.kv[rows]
    sub.q_req = np.asarray([remap[int(b)] for b in wl.q_req[qs]], np.int32)
    sub.q_pos = wl.q_pos[qs].copy()
    sub.hidden, sub.q_idx, sub.q_mla = wl.hidden[qs], wl.q_idx[qs], wl.q_mla[qs]
    return sub


def oracle_queries(wl, n: int):
    """A bounded sample: the first n queries, spread over the batch's requests."""
    n = max(1, min(n, wl.Q))
    return np.unique(np.linspace(0, wl.Q - 1, n).round().astype(int))


def time_oracle(wl, min_seconds: float, n_q: int):
    """The oracle pipeline on a sample of n_q queries (and the requests they read),
    repeated until min_seconds elapse. Returns (queries/s, cores, sample description)."""
    import oracle as O
    qs = oracle_queries(wl, n_q)
    sub = sample_workload(wl, qs)
    cores = os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:
        O.pipeline(sub, threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return (len(qs) * reps / el, cores,
            f"{len(qs)} of {wl.Q} queries with their {sub.B} requests, {reps} passes, {el:.1f} s")


def reference_arm(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # one query (with its request) per step keeps --steps K within a few minutes at the
    # K the GPU arm uses (about 27 ms a step on 16 host cores for a decode query)
    n_q = 2 if args.steps + args.warmup <= 200 else 1
    import oracle as O
    qs = oracle_queries(wl, n_q)
    sub = sample_workload(wl, qs)
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        O.pipeline(sub, threads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.pipeline(sub, threads=cores)
    el = time.perf_counter() - t0
    qps = len(qs) * args.steps / el
    sample = f"{len(qs)} of {wl.Q} queries (with their {sub.B} requests) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": sample},
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def stage_times(steps, stream, names, n_rep):
    """Mean device time (ms) of each stage on its own. Each stage is bracketed by events
    and preceded by a short device sleep, so the CPU has enqueued the event/kernel/event
    triple before the GPU reaches it and no host gap falls inside a bracket."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
           for _ in range(n_rep)]
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for r in range(n_rep):
            s = steps[r % len(steps)]
            for i, n in enumerate(names):
                torch.cuda._sleep(200_000)
                evs[r][2 * i].record(stream)
                getattr(s, n)(stream)
                evs[r][2 * i + 1].record(stream)
    stream.synchronize()
    return {n: statistics.mean(evs[r][2 * i].elapsed_time(evs[r][2 * i + 1]) for r in range(n_rep))
            for i, n in enumerate(names)}


def stage_times_back_to_back(steps, stream, names, n_launch):
    """Device time (ms) per launch of each stage run n_launch times back to back over
    the rotating input sets, between one pair of events (launch latency and the
    programmatic-dependent-launch overlap of consecutive launches as in a pipeline).
    A device sleep first lets the CPU enqueue every launch before the GPU reaches them."""
    import torch
    out = {}
    for n in names:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            torch.cuda._sleep(4_000_000)
            e0.record(stream)
            for r in range(n_launch):
                getattr(steps[r % len(steps)], n)(stream)
            e1.record(stream)
        stream.synchronize()
        out[n] = e0.elapsed_time(e1) / n_launch
    return out


def timed_replays(graphs, stream, steps, world):
    """Device time (ms, max over ranks) of `steps` graph replays, and the wall-clock
    window (perf_counter) of the timed region."""
    import torch
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(2_000_000)           # keeps the GPU busy while the CPU enqueues
        ev0.record(stream)
        t0 = time.perf_counter()
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        ev1.record(stream)
    stream.synchronize()
    t1 = time.perf_counter()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(ev0.elapsed_time(ev1), world), t0, t1


def measure(args, wl, dev, rank, world, local, headline: bool) -> dict:
    """One workload on this rank's GPU; returns the JSON line (rank 0) or None."""
    import torch
    from sparse_attention_indexer_head_b200 import binding as B
    from sparse_attention_indexer_head_b200.pipeline import (QUERY_INPUTS, DecodeStep,
                                                             StreamedDecode, host_tensors)
    fused = {"fused": True, "staged": False, "auto": "auto"}[args.path]
    all_bytes = algorithmic_bytes(wl)
    host = host_tensors(wl)
    steps = [DecodeStep(wl, device=str(dev), inputs=host, fused_indexer=fused)]
    names = steps[0].stages()
    steps_fused = steps[0].fused
    per_stage_bytes = {n: all_bytes[n] for n in names}
    step_bytes = sum(per_stage_bytes.values())
    n_sets = input_sets(step_bytes, args.sets)
    steps += [DecodeStep(wl, device=str(dev), inputs=host, fused_indexer=fused)
              for _ in range(n_sets - 1)]
    stream = torch.cuda.Stream(device=dev)
    clocks = ClockSampler(local) if rank == 0 else None

    # Warm every set once eagerly (sets kernel attributes), then capture one graph per set.
    with torch.cuda.stream(stream):
        for s in steps:
            s.run()
    stream.synchronize()
    graphs = []
    for s in steps:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            s.run()
        graphs.append(g)
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % len(graphs)].replay()
    stream.synchronize()
    if clocks:
        clocks.wait_first()
    ms_total, t_wall0, t_wall1 = timed_replays(graphs, stream, args.steps, world)
    ms_per_step = ms_total / args.steps
    value = replica_throughput(wl.Q, world, args.steps, ms_total / 1e3)
    clk = clocks.summary(t_wall0, t_wall1) if clocks else None

    n_rep = max(5, min(args.steps, 100))
    stage_ms = stage_times(steps, stream, names, n_rep)
    stage_b2b_ms = stage_times_back_to_back(steps, stream, names, 30)

    incremental = None
    if headline:
        # Incremental decode step: the cache update stores each request's new indexer
        # row and recomputes only the pools holding it, in place of the full compress
        # (the pooled keys already hold the compress result of the cache).
        for s in steps:
            s.stage_new_tokens()
        with torch.cuda.stream(stream):
            for s in steps:
                s.run_incremental(stream)
        stream.synchronize()
        inc_graphs = []
        for s in steps:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                s.run_incremental()
            inc_graphs.append(g)
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                inc_graphs[i % len(inc_graphs)].replay()
        stream.synchronize()
        inc_ms, _, _ = timed_replays(inc_graphs, stream, args.steps, world)
        inc_names = ["indexer_store", "kpool_compress_tokens"]
        inc_stage = stage_times(steps, stream, inc_names, n_rep)
        incremental = {
            "value": replica_throughput(wl.Q, world, args.steps, inc_ms / 1e3), "unit": "queries/s",
            "ms_per_step": inc_ms / args.steps, "steps": args.steps,
            "gpu_launches": steps[0].kernels_per_step_incremental() * args.steps,
            "stage_us": {k: 1e3 * v for k, v in inc_stage.items()},
            "new_rows_per_step": steps[0].new["n"],
            "path": "dsa_indexer_store of each request's new row -> dsa_kpool_compress_tokens "
                    "over its pools -> the indexer stage(s) and the MLA as in the step above",
        }
        del inc_graphs

    launches = steps[0].kernels_per_step() * args.steps
    del graphs, steps
    torch.cuda.synchronize()

    # End to end through the public API with host buffers: StreamedDecode copies each
    # step's query inputs from pinned host memory, runs the step and copies its output
    # back, consecutive steps on E2E_SLOTS streams; every step's output is read on the
    # host inside the timed region, step i-(E2E_SLOTS-1)'s once step i is enqueued, so
    # one step's input copy, another's kernels and a third's output copy overlap. The
    # loop runs at least --e2e-seconds, whatever --steps is, so it measures steady state.
    sd = StreamedDecode(wl, device=str(dev), slots=E2E_SLOTS, inputs=host, fused_indexer=fused)
    for k in range(E2E_SLOTS):
        sd.write_inputs(k, {n: host[n] for n in QUERY_INPUTS})
    h2d = sd.nbytes
    d2h = sd.out_host[0].numel() * sd.out_host[0].element_size()
    lag = E2E_SLOTS - 1
    for i in range(4):
        sd.result(sd.submit())
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(8):
        sd.result(sd.submit())
    per = (time.perf_counter() - t0) / 8
    e2e_steps = int(max(3, args.steps, min(200000, args.e2e_seconds / max(per, 1e-6))))
    e2e_steps = int(max_over_ranks(float(e2e_steps), world))
    barrier(world)
    t0 = time.perf_counter()
    base = sd.submitted
    for i in range(e2e_steps):
        sd.submit()
        if i >= lag:
            sd.result(base + i - lag)
    for i in range(max(0, e2e_steps - lag), e2e_steps):
        sd.result(base + i)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world)
    e2e_value = replica_throughput(wl.Q, world, e2e_steps, e2e_s)
    del sd

    if clocks:
        clocks.stop()
    if rank != 0:
        return None

    # ---- roofline of the dominant kernel (the stage with the longest device time)
    hbm, tflops, peak_kind = peaks()
    dom = max(stage_ms, key=stage_ms.get)
    t_dom = stage_ms[dom] * 1e-3
    flops = mla_flops(wl)
    # The MLA is bound by the tensor cores when its flops take longer at the bf16 peak
    # than its bytes at the HBM peak (chunked prefill); every other stage by HBM.
    mla_tensor = flops / (tflops * 1e12) > per_stage_bytes["sparse_mla"] / (hbm * 1e9)
    if dom == "sparse_mla" and mla_tensor:
        achieved = flops / t_dom / 1e12
        b2b = flops / (stage_b2b_ms[dom] * 1e-3) / 1e12
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": tflops,
                    "unit": "TFLOP/s", "frac": achieved / tflops, "traffic": None,
                    "peak_kind": peak_kind + " bf16 dense (burst: the stage is timed alone)",
                    "algorithmic_flops": flops,
                    "achieved_back_to_back": b2b, "frac_back_to_back": b2b / tflops}
    else:
        achieved = per_stage_bytes[dom] / t_dom / 1e9
        b2b = per_stage_bytes[dom] / (stage_b2b_ms[dom] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                    "unit": "GB/s", "frac": achieved / hbm,
                    "traffic": traffic_for(dom, STAGE_SOURCE[dom], args.config_key),
                    "peak_kind": peak_kind, "algorithmic_bytes": per_stage_bytes[dom],
                    "achieved_back_to_back": b2b, "frac_back_to_back": b2b / hbm}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        qps, cores, sample = time_oracle(wl, args.cpu_seconds, args.cpu_queries)
        cpu = {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "path": "fused" if steps_fused else "staged",
                   "global_batch": wl.Q * world,
                   "seq_len": int(max(wl.lengths)), "parallelism": f"replicas x{world}",
                   "l2": f"inputs rotated over {n_sets} device-resident sets "
                         f"({n_sets * step_bytes / 1e9:.2f} GB > L2)",
                   "timing": "CUDA graph replays, CUDA events, max over ranks"},
        "achieved_gbs": step_gbs, "hbm_frac": step_gbs / hbm,
        "algorithmic_bytes_per_step": step_bytes,
        "mla_flops_per_step": flops,
        "stage_us": {k: 1e3 * v for k, v in stage_ms.items()},
        "stage_us_back_to_back": {k: 1e3 * v for k, v in stage_b2b_ms.items()},
        "stage_timing": ("stage_us: each stage alone between events after a device sleep, "
                         "launch latency included (the roofline's achieved and frac); "
                         "stage_us_back_to_back: 30 launches of the stage back to back over "
                         "the rotating input sets between one event pair, per launch"),
        "stage_bytes": per_stage_bytes,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "seconds": e2e_s,
                "path": "StreamedDecode: per step one graph replay of H2D of the packed pinned "
                        "query inputs -> the step's ABI calls -> D2H of out, consecutive steps "
                        f"on {E2E_SLOTS} streams; each step's output read on the host "
                        f"{E2E_SLOTS - 1} submissions later"},
        "gpu_launches": launches,
        "incremental": incremental,
        "clocks": clk,
        "device_error": B.dsa_device_status(reset=True),
    }


def gpu_arm(args, names):
    import torch
    rank, world, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from sparse_attention_indexer_head_b200 import build as _build
    if not os.path.exists(os.path.join(ROOT, "sparse_attention_indexer_head_b200", "libdsa.so")):
        _build.build()
    from sparse_attention_indexer_head_b200 import workloads as W
    for name in names:
        args.config_key = name
        # weak scaling: each rank draws its own batch (seed = rank)
        line = measure(args, W.make(name, seed=rank), dev, rank, world, local,
                       headline=(name == "batched"))
        if line is not None:
            print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="batched",
                    choices=["tiny", "batched", "ragged", "long", "prefill", "all"])
    ap.add_argument("--sets", type=int, default=0, help="input sets to rotate (0: enough for L2)")
    ap.add_argument("--path", default="auto", choices=["auto", "fused", "staged"],
                    help="fused: compress -> dsa_indexer_select -> MLA; staged: the five calls; "
                         "auto: fused for decode-sized batches")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-queries", type=int, default=16)
    ap.add_argument("--e2e-seconds", type=float, default=0.5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    names = ["tiny", "batched", "ragged", "long", "prefill"] if args.config == "all" else [args.config]

    from sparse_attention_indexer_head_b200 import workloads as W
    if args.impl == "reference":
        return reference_arm(args, W.make(names[0], seed=0))
    return gpu_arm(args, names)


if __name__ == "__main__":
    sys.exit(main())
