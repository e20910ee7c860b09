"""The bench's multi-rank path on the host: two gloo ranks (world size 2).

The bench runs one independent replica per GPU (no data-path collective).  Its
host logic is what these tests cover, on CPU processes: every rank takes the
same collective steps, the step time is the maximum over the ranks, the value
is the whole job's throughput, and the reference arm does its work on rank 0
only while the other ranks leave without any.
"""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        slowest = bench.max_over_ranks(1.0 + rank, world)     # rank r's "step time"
        bench.barrier(world)
        value = bench.aggregate(100.0, slowest, world)          # 100 units per rank per step
        # the reference arm: rank 0 alone works; the others return at once
        class A:
            steps, warmup, ref_seconds = 1, 0, 0.01
        ref_done = None
        if rank != 0:
            bench.run_reference(A, world, rank)
            ref_done = "returned"
        q.put((rank, slowest, value, ref_done))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=150) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_rank = {r: (s, v, ref) for r, s, v, ref in got}
    for r in range(world):
        slowest, value, _ = by_rank[r]
        assert slowest == 2.0                                   # the max over ranks, on every rank
        assert value == pytest.approx(world * 100.0 / 2e-3)     # whole-job units per second
    assert by_rank[1][2] == "returned"


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate(10.0, 2.0, 1) == pytest.approx(5000.0)


def test_percentile_helper():
    import bench
    ms = [i / 1000.0 for i in range(1, 102)]        # 1..101 µs
    p10, p50, p90 = bench.pcts(ms)
    assert p50 == pytest.approx(51.0)
    assert p10 == pytest.approx(11.0) and p90 == pytest.approx(91.0)
    assert bench.pcts([0.002]) == [2.0, 2.0, 2.0]
