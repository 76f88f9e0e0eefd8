"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
each rank gets its own seeded workload (replicas, no data exchange), the
timed region is the max over ranks, and the job value counts every rank's
bytes over the slowest rank's time."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        t = bench.reduce_max(local_ms, world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        out.put((rank, t, seeds))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, seeds in got:
        assert t == 20.0  # the slowest rank's time, on every rank
        assert len(set(seeds)) == 2  # each rank quantizes its own data
    # weak scaling: two ranks move twice the bytes in the slowest rank's time
    assert bench.job_gbs(2, 1e9, 10, 20.0) == pytest.approx(2 * bench.job_gbs(1, 1e9, 10, 20.0))


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_gbs(1, 2e9, 4, 8.0) == pytest.approx(1000.0)
