"""bench.py's multi-rank host logic (replicas only: a barrier and the max of
the ranks' timings, no data exchange), run as two gloo ranks on the CPU."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    assert bench.dist_setup() == (world, rank, rank)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        slowest = bench.max_over_ranks(times[rank])
        rate = bench.whole_job_rate(world, 16 * 100, slowest)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    times = [0.75, 1.25]   # seconds per rank for 100 steps of 16 tokens
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, slowest, rate in got:
        assert slowest == pytest.approx(1.25)                  # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 16 * 100 / 1.25)      # all ranks' tokens over that time


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(1, 1600, 0.5) == pytest.approx(3200.0)
