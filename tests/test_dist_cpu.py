"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): every rank runs
its own replica of the batch, timings are combined as the max over ranks and
throughput counts the work of all ranks."""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r pretends its step took 10*(r+1) ms and its attention 3+r ms
    ms, att = bench.max_over_ranks([10.0 * (rank + 1), 3.0 + rank])
    gbs = bench.whole_job_gbs(1e9, ms, world)
    results[rank] = (ms, att, gbs)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world = 2
    port = 29500 + (os.getpid() % 1000)
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        ms, att, gbs = results[rank]
        assert ms == 20.0 and att == 4.0
        assert gbs == pytest.approx(2 * 1e9 / 0.020 / 1e9)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_gbs(2e9, 1000.0, 1) == pytest.approx(2.0)
