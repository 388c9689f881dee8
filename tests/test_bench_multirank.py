"""The benchmark's N > 1 host logic on CPU: two ranks over gloo.

bench.py runs N independent block replicas (one process per GPU, no
collective on the data path); across ranks it only takes the slowest rank's
time (one MAX all-reduce) and reports the whole job's throughput, and the
reference arm runs on rank 0 alone.  These tests exercise exactly that logic
with world size 2 on the host (NCCL on the GPU uses the same calls)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 is the slow one for the first value, rank 0 for the second
        times = [10.0 + 5.0 * rank, 7.0 - 3.0 * rank]
        got = bench.max_over_ranks(times, torch.device("cpu"))
        rate = bench.job_rate(2.0e12, world, 4, got[0])
        out[rank] = (got, rate)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_two_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        got, rate = out[rank]
        assert got == [15.0, 7.0]  # every rank sees the slowest rank's times
        # 2 ranks x 2 TFLOP x 4 steps in 15 ms
        assert rate == pytest.approx(2 * 2.0 * 4 / 15e-3)


def test_single_rank_is_a_no_op():
    assert bench.max_over_ranks([3.0, 4.0], torch.device("cpu")) == [3.0, 4.0]
    assert bench.job_rate(1e12, 1, 10, 1000.0) == pytest.approx(10.0)


def test_reference_arm_runs_on_rank_0_only():
    class Args:
        config = "1024px"
        steps = 1
        warmup = 0
    # any rank but 0 returns at once with status 0 and does no work
    assert bench.run_reference(Args(), rank=1, world=2) == 0
