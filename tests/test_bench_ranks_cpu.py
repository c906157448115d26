"""bench.py's multi-rank arithmetic on two gloo ranks (CPU): the step time is the slowest
rank's, and the job's throughput counts every rank's units (weak scaling)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [1.25, 2.5][rank]
        ms = bench.max_over_ranks(ms_local, world)
        q.put((rank, ms, bench.job_value(world, 4098, ms)))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_sets_the_time_and_units_add_up():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in got:
        assert ms == 2.5
        assert value == pytest.approx(2 * 4098 / 2.5e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.job_value(1, 100, 2.0) == pytest.approx(50000.0)
