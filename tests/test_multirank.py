"""Multi-rank logic of the benchmark on CPU (gloo, world size 2).

Each rank runs its own layer call (weak scaling, no data-path collective); the
job's time is the slowest rank's, and the throughput counts every rank's units.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ret):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.5 + rank                       # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, torch.device("cpu"))
        value, tok = bench.job_throughput(1.5e12, 32760, ms_max, world)
        ret[rank] = (ms_max, value, tok)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    mgr = mp.Manager()
    ret = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), ret), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms_max, value, tok = ret[r]
        assert ms_max == 2.5
        assert value == pytest.approx(1.5e12 * 2 / 2.5e-3 / 1e12)
        assert tok == pytest.approx(32760 * 2 / 2.5e-3)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.0, torch.device("cpu")) == 3.0
    assert bench.job_throughput(1e12, 100, 1.0, 1) == (1000.0, 100000.0)
