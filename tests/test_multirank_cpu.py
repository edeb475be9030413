"""Multi-rank host logic of the benchmark on CPU: gloo process group, world size 2.

The library's data path has no collective (heads are independent, N GPUs run N
replicas); what crosses ranks is the timing: every rank reports its own time and
the job's time is the slowest rank's.  These tests run two gloo ranks on the CPU.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [3.0, 7.5][rank]
        ms_max = bench.max_over_ranks(local)
        value = bench.job_throughput(world, 1000, 10, ms_max)
        results[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value():
    world = 2
    with mp.get_context("spawn").Manager() as man:
        results = man.dict()
        mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    assert res[0] == res[1]
    ms_max, value = res[0]
    assert ms_max == 7.5
    assert value == pytest.approx(2 * 1000 * 10 / 7.5e-3)


def test_single_process_needs_no_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.job_throughput(1, 8196, 50, 125.0) == pytest.approx(8196 * 50 / 0.125)
