"""The bench's multi-rank path on CPU: two gloo ranks, no GPU.

bench.py --gpus N runs one replica per rank (each rank its own batch, seed =
rank) with no collective on the data path; ranks meet only at barriers and at
the max-over-ranks reduction of the step time. Those host-side pieces are what
this file exercises, over the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    import bench
    from sparse_attention_indexer_head_b200 import workloads as W

    r, w, local = bench.dist_setup("gloo")
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    # the step time every rank reports is the slowest rank's
    t = bench.max_over_ranks(10.0 + rank, w, device="cpu")
    # each replica draws its own batch
    wl = W.make("tiny", seed=rank)
    digest = float(np.asarray(wl.q_idx, dtype=np.float64).sum())
    digests = [None] * w
    dist.all_gather_object(digests, digest)
    bench.barrier(w)
    dist.destroy_process_group()
    out.put((rank, t, digests))


def test_two_gloo_ranks_reduce_time_and_draw_distinct_batches():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = dict((r, (t, d)) for r, t, d in results)
    assert by_rank[0][0] == by_rank[1][0] == 11.0          # max over ranks
    d0, d1 = by_rank[0][1]
    assert d0 != d1                                        # seed = rank: different batches
    assert by_rank[0][1] == by_rank[1][1]                  # every rank sees the same set


def test_replica_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 16 queries per rank, 8 ranks, 100 steps in 0.5 s (the slowest rank's time)
    assert bench.replica_throughput(16, 8, 100, 0.5) == pytest.approx(25600.0)
    assert bench.replica_throughput(16, 1, 100, 0.5) == pytest.approx(3200.0)
