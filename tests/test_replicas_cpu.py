"""The multi-GPU plumbing of bench.py on CPU: world-size-2 gloo ranks.

Multi-GPU runs are independent replicas (the path needs no exchange between
GPUs); what the ranks share is the barrier around the timed region, the
max-over-ranks time and the whole-job aggregate, and, for the reference arm,
that rank 0 alone works.  Ranks are spawned processes on 127.0.0.1.
"""

from __future__ import annotations

import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        dist.barrier()
        times = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world, "cpu")
        value = bench.whole_job_gbps(world, 1e9, 4, times[0])
        # the reference arm: rank 0 alone works, the others return at once
        worked = []

        class _Args:
            steps = 0
            warmup = 0

        if rank != 0:
            bench.run_reference(_Args(), rank, world)
            worked.append(False)
        dist.barrier()
        q.put((rank, times, value, worked))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_aggregate():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(2):
        rank, times, value, worked = q.get(timeout=120)
        results[rank] = (times, value, worked)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        times, value, _ = results[rank]
        assert times == [2.0, 10.0]               # element-wise max over the two ranks
        assert value == pytest.approx(2 * 1e9 * 4 / 2.0 / 1e9)
    assert results[1][2] == [False]               # rank 1 returned from the reference arm


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.5, 1], 1, "cpu") == [3.5, 1.0]
    assert bench.whole_job_gbps(1, 2e9, 10, 4.0) == pytest.approx(5.0)
