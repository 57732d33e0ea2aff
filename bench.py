#!/usr/bin/env python3
"""Benchmark of the DSA decode hot path on B200 (one JSON line on rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path -- head gate, kpool_compress (+k_norm),
index_scores, top-k + expand, sparse NoPE MLA -- over one batch of the
batched-decode workload: 16 requests x 8192 cached tokens (left pad U{0..64}),
kpool 4 (2048 pools), 512 pools (2048 tokens) selected per query, 64 MLA heads
over a 512-wide NoPE latent. Inputs are seeded synthetic arrays of those shapes.

Timing: CUDA graphs of the six kernel launches, replayed over 3 device-resident
input sets (about 0.6 GB, larger than the 126 MB L2) so no step reads another
step's inputs from L2; CUDA events on the launching stream with a barrier and
a synchronize on both sides; the max over ranks. Under torchrun each rank runs
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
import subprocess
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
    mla = int((n_sel * kp * L * 2).sum() + Q * (wl.hm * L * 2 * 2 + 4 * wl.out_width + 4 * wl.hm + 4))
    return dict(head_gate=gate, kpool_compress=compress, index_scores=scores,
                topk_expand=topk, sparse_mla=mla)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (SM clock, reasons) in a background thread."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        inside = [s for t, s in self.samples if t0 <= t <= t1]
        near = inside or [s for t, s in self.samples if t0 - 1.0 <= t <= t1 + 1.0]
        if not near:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"],
                    "samples_in_region": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(s[2]) for s in near if num(s[2]) is not None]
        mx = [num(s[3]) for s in near if num(s[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in near for i in range(4)
                          if len(s) > 6 + i and s[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples_in_region": len(inside)}


# ----------------------------------------------------------------------------- helpers
def peaks():
    try:
        with open(PEAKS_FILE) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(kernel_file: str) -> str:
    csrc = os.path.join(ROOT, "sparse_attention_indexer_head_b200", "csrc")
    h = hashlib.sha256()
    for name in ("common.cuh", kernel_file):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, kernel_file: str, units_scale: float = 1.0):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    try:
        with open(TRAFFIC_FILE) as fh:
            t = json.load(fh)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if t.get("source_sha") != kernel_source_sha(kernel_file):
        return None
    return float(t["dram_bytes_per_launch"]) * units_scale


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


# ----------------------------------------------------------------------------- oracle timing
def time_oracle(wl, min_seconds: float, n_req: int):
    """The oracle pipeline on the first n_req requests (one query each), repeated until
    min_seconds elapse. Returns (queries/s, cores, sample description)."""
    import oracle as O
    from sparse_attention_indexer_head_b200 import workloads as W
    sub = W.build(wl.name + " (oracle sample)", lengths=wl.lengths[:n_req], pads=wl.pads[:n_req],
                  kpool=wl.kpool, max_pools=wl.max_pools, select_k=wl.select_k, hm=wl.hm,
                  q_req=list(range(n_req)), q_pos=[t - 1 for t in wl.lengths[:n_req]],
                  seed=wl.seed)
    cores = os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:
        O.pipeline(sub, threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    return n_req * reps / el, cores, f"{n_req} of {wl.B} requests (1 query each), {reps} passes, {el:.1f} s"


def reference_arm(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # one request (one decode query) per step keeps --steps K within a few minutes
    # at the K the GPU arm uses (about 27 ms a step on 16 host cores)
    n_req = 2 if args.steps + args.warmup <= 200 else 1
    import oracle as O
    from sparse_attention_indexer_head_b200 import workloads as W
    sub = W.build(wl.name, lengths=wl.lengths[:n_req], pads=wl.pads[:n_req], kpool=wl.kpool,
                  max_pools=wl.max_pools, select_k=wl.select_k, hm=wl.hm,
                  q_req=list(range(n_req)), q_pos=[t - 1 for t in wl.lengths[:n_req]], seed=0)
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        O.pipeline(sub, threads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.pipeline(sub, threads=cores)
    el = time.perf_counter() - t0
    qps = n_req * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample": f"{n_req} of {wl.B} requests per step"},
        "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_req} of {wl.B} requests (1 query each) per step"},
        "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def gpu_arm(args, wl_fn):
    import torch
    rank, world, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from sparse_attention_indexer_head_b200 import build as _build
    if not os.path.exists(os.path.join(ROOT, "sparse_attention_indexer_head_b200", "libdsa.so")):
        _build.build()
    from sparse_attention_indexer_head_b200 import binding as B
    from sparse_attention_indexer_head_b200.pipeline import QUERY_INPUTS, DecodeStep, host_tensors

    wl = wl_fn(rank)
    per_stage_bytes = algorithmic_bytes(wl)
    step_bytes = sum(per_stage_bytes.values())
    host = host_tensors(wl)
    steps = [DecodeStep(wl, device=str(dev), inputs=host) for _ in range(args.sets)]
    stream = torch.cuda.Stream(device=dev)

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

    clocks = ClockSampler(local) if rank == 0 else None

    # ---- warm-up
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % len(graphs)].replay()
    stream.synchronize()

    # ---- timed region: K graph replays
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(2_000_000)           # keeps the GPU busy while the CPU enqueues
        ev0.record(stream)
        t_wall0 = time.time()
        for i in range(args.steps):
            graphs[i % len(graphs)].replay()
        ev1.record(stream)
    stream.synchronize()
    t_wall1 = time.time()
    torch.cuda.synchronize()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms_total = max_over_ranks(ms_local, world)
    ms_per_step = ms_total / args.steps
    value = replica_throughput(wl.Q, world, args.steps, ms_total / 1e3)
    clk = clocks.summary(t_wall0 - 0.05, t_wall1 + 0.05) if clocks else None

    # ---- per-stage device time. Each stage is bracketed by events and preceded by a
    # short device sleep, so the CPU has enqueued the event/kernel/event triple before
    # the GPU reaches it and no host gap falls inside a bracket.
    names = ["head_gate", "kpool_compress", "index_scores", "topk_expand", "sparse_mla"]
    n_rep = max(5, min(args.steps, 100))
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
    stage_ms = {n: statistics.mean(evs[r][2 * i].elapsed_time(evs[r][2 * i + 1])
                                   for r in range(n_rep))
                for i, n in enumerate(names)}

    # ---- incremental decode step: the cache update stores each request's new
    # indexer row and recomputes only the pools holding it, in place of the full
    # compress (the pooled keys already hold the compress result of the cache).
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
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        torch.cuda._sleep(2_000_000)
        ev0.record(stream)
        for i in range(args.steps):
            inc_graphs[i % len(inc_graphs)].replay()
        ev1.record(stream)
    stream.synchronize()
    barrier(world)
    inc_ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    inc_names = ["indexer_store", "kpool_compress_tokens"]
    inc_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_rep)]
    with torch.cuda.stream(stream):
        for r in range(n_rep):
            s = steps[r % len(steps)]
            for i, n in enumerate(inc_names):
                torch.cuda._sleep(200_000)
                inc_evs[r][2 * i].record(stream)
                getattr(s, n)(stream)
                inc_evs[r][2 * i + 1].record(stream)
    stream.synchronize()
    inc_stage_us = {n: 1e3 * statistics.mean(inc_evs[r][2 * i].elapsed_time(inc_evs[r][2 * i + 1])
                                             for r in range(n_rep))
                    for i, n in enumerate(inc_names)}
    incremental = {
        "value": replica_throughput(wl.Q, world, args.steps, inc_ms / 1e3), "unit": "queries/s",
        "ms_per_step": inc_ms / args.steps, "steps": args.steps,
        "gpu_launches": steps[0].kernels_per_step_incremental() * args.steps,
        "stage_us": inc_stage_us, "new_rows_per_step": steps[0].new["n"],
        "path": "dsa_indexer_store of each request's new row -> dsa_kpool_compress_tokens "
                "over its pools -> gate, scores, top-k, MLA as in the step above",
    }
    del inc_graphs

    # ---- end to end through the public API with host buffers: StreamedDecode copies
    # each step's query inputs from pinned host memory, runs the step and copies its
    # output back, with consecutive steps on two streams; every step's output is
    # read on the host (step i-1's while step i is enqueued) inside the timed region.
    from sparse_attention_indexer_head_b200.pipeline import StreamedDecode
    sd = StreamedDecode(wl, device=str(dev), slots=2, inputs=host)
    for k in range(2):
        sd.write_inputs(k, {n: host[n] for n in QUERY_INPUTS})
    h2d = sd.nbytes
    d2h = sd.out_host[0].numel() * sd.out_host[0].element_size()
    e2e_steps = max(3, min(args.steps, 2000))
    for i in range(4):
        sd.result(sd.submit())
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    base = sd.submitted
    for i in range(e2e_steps):
        sd.submit()
        if i >= 1:
            sd.result(base + i - 1)
    sd.result(base + e2e_steps - 1)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world)
    e2e_value = replica_throughput(wl.Q, world, e2e_steps, e2e_s)
    del sd

    if clocks:
        clocks.stop()
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # ---- roofline of the dominant kernel (kpool_compress)
    peak, peak_kind = peaks()
    dom = "kpool_compress"
    achieved = per_stage_bytes[dom] / (stage_ms[dom] * 1e-3) / 1e9
    traffic = traffic_for(dom, "kpool_compress.cuh")
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                "peak_kind": peak_kind, "algorithmic_bytes": per_stage_bytes[dom]}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        qps, cores, sample = time_oracle(wl, args.cpu_seconds, args.cpu_requests)
        cpu = {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
               "sample": sample}

    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32",
        "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": wl.Q * world,
                   "seq_len": int(max(wl.lengths)), "parallelism": f"replicas x{world}",
                   "l2": f"inputs rotated over {args.sets} device-resident sets "
                         f"({args.sets * step_bytes / 1e9:.2f} GB > L2)",
                   "timing": "CUDA graph replays, CUDA events, max over ranks"},
        "achieved_gbs": step_gbs, "hbm_frac": step_gbs / peak,
        "algorithmic_bytes_per_step": step_bytes,
        "stage_us": {k: 1e3 * v for k, v in stage_ms.items()},
        "stage_bytes": per_stage_bytes,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "StreamedDecode: per step one graph replay of H2D of the packed pinned "
                        "query inputs -> the five ABI calls -> D2H of out, consecutive steps "
                        "on two streams; each step's output read on the host"},
        "gpu_launches": steps[0].kernels_per_step() * args.steps,
        "incremental": incremental,
        "clocks": clk,
        "device_error": B.dsa_device_status(reset=True),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sets", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-requests", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from sparse_attention_indexer_head_b200 import workloads as W
    if args.impl == "reference":
        return reference_arm(args, W.batched(seed=0))
    # weak scaling: each rank draws its own batch (seed = rank)
    return gpu_arm(args, lambda rank: W.batched(seed=rank))


if __name__ == "__main__":
    sys.exit(main())
