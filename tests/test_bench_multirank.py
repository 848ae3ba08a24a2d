"""bench.py's multi-rank host logic on CPU with gloo, world size 2.

Every rank runs its own batch (replicas); the job's step time is the slowest
rank's, and the job's throughput counts every rank's work.
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local = [100.0 + 50.0 * rank, 20.0 + rank, 80.0 + 49.0 * rank]   # rank 1 is slower
    value, t = bench.aggregate(local, world, flops_step=1e12, steps=10, pg=dist)
    out[rank] = (value, t)
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_takes_max_over_ranks_and_counts_all_work():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        value, t = out[rank]
        assert t == [150.0, 21.0, 129.0]                 # elementwise max over ranks
        assert value == pytest.approx(2 * 1e12 * 10 / 0.150 / 1e12)


def test_aggregate_single_process():
    import bench
    value, t = bench.aggregate([200.0, 50.0, 150.0], 1, 2e12, 4)
    assert t == [200.0, 50.0, 150.0]
    assert value == pytest.approx(2e12 * 4 / 0.2 / 1e12)
