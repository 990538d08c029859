"""The multi-rank plumbing of bench.py (replicas: a barrier and the max over
ranks of the timed region) on world_size 2 with gloo on the CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        barrier, max_over_ranks = bench.rank_ops(torch, dist, world, torch.device("cpu"))
        barrier()
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        out[rank] = max_over_ranks(ms)
        barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_gloo():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork: CUDA may be initialised in this process
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_needs_no_process_group():
    barrier, max_over_ranks = bench.rank_ops(torch, dist, 1, torch.device("cpu"))
    barrier()
    assert max_over_ranks(3.5) == 3.5


def test_whole_job_value_is_weak_scaling_aggregate():
    # two ranks each streaming 1 GB per step for 10 steps in (slowest) 1 s -> 20 GB/s
    assert bench.whole_job_gbs(2, 10 ** 9, 10, 1000.0) == pytest.approx(20.0)
    assert bench.whole_job_gbs(1, 10 ** 9, 10, 1000.0) == pytest.approx(10.0)


def test_cold_rotation_exceeds_three_l2():
    l2 = 126 * 1024 * 1024
    for nbytes in (2560 * 640 // 4, 2560 * 6912 // 4, 8192 * 28672 // 4):
        n = bench.cold_copies(l2, nbytes)
        assert n * nbytes >= 3 * l2 and (n - 1) * nbytes < 3 * l2 or n == 2
    assert bench.cold_copies(l2, 2560 * 6912 // 4) == 90
    assert bench.cold_copies(l2, 8192 * 28672 // 4) == 7
