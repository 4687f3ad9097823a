"""N > 1 host logic on CPU: two gloo ranks, independent instances, max-over-ranks timing.

The attention path shards by (b, h) with no data-path collective, so the only
multi-rank logic is on the host: each rank owns a distinct seeded instance, and
the step time is the max over ranks. Runs as two spawned processes on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local = [10.0 + rank * 5.0, 3.0 - rank]  # rank 1 is slower on the first, faster on the second
        got = bench.reduce_max(local, world, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed("c2", rank))
        out[rank] = (got, seeds, bench.job_throughput(1e12, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_seeds():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        got, seeds, tput = out[r]
        assert got == [15.0, 3.0]
        assert len(set(seeds)) == world  # independent instances
        assert tput == pytest.approx(1e12 * world / 15e-3 / 1e12)
