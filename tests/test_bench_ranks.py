"""Multi-rank accounting of bench.py on CPU: two gloo ranks (replicas) agree on the
slowest rank's time, and the whole-job value counts the work of both ranks."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        tot = bench.max_over_ranks(my_ms, dist, "cpu")
        q.put((rank, tot, bench.job_value(world, 4, 1e12, tot)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tot, val in res:
        assert tot == 15.0                       # max over ranks
        assert val == pytest.approx(2 * 4 * 1e12 / 15e-3 / 1e12)  # both ranks' work / slowest time


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.job_value(1, 10, 2e12, 20.0) == pytest.approx(1000.0)
