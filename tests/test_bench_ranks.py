"""The multi-process side of bench.py on CPU: two gloo ranks, each with its
own replica timing; the job's time is the slowest rank's and its throughput
counts every rank's tokens."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = (ms, bench.job_throughput(world, 2048, ms / 4))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # 4 steps in 15 ms on each of 2 replicas of 2,048 tokens
    assert res[0][1] == pytest.approx(2 * 2048 / (15.0 / 4 / 1e3))


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.job_throughput(1, 2048, 0.5) == pytest.approx(4.096e6)
