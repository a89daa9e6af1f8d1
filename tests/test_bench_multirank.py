"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (127.0.0.1) check
that the whole-job rate divides every rank's units by the slowest rank's time,
and that every rank takes the same collective steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_seconds = 1.0 + rank                        # rank 1 is the slowest
        rate = bench.whole_job_rate(100.0, local_seconds, world, dist, "cpu")
        mx = bench.max_over_ranks(local_seconds, dist, "cpu")
        q.put((rank, rate, mx))
    finally:
        dist.destroy_process_group()


def test_whole_job_rate_uses_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, rate, mx in got:
        assert mx == 2.0
        assert rate == pytest.approx(world * 100.0 / 2.0)


def test_single_process_needs_no_group():
    assert bench.whole_job_rate(50.0, 2.0, 1, None, "cpu") == 25.0
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
