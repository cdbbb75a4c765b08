"""The bench's multi-rank host logic on CPU: two ranks over gloo (world size 2).

The path runs replicas (no collective on the data path); the only cross-rank
steps are the barrier and the max-over-ranks of the timed durations, and
the whole-job rate is all ranks' work over the slowest rank's time."""

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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        # each rank "measured" a different duration; every rank must see the largest
        slowest = bench.max_over_ranks(1.0 + rank, world)
        rate = bench.job_throughput(100.0, world, slowest)
        out[rank] = (slowest, rate)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        slowest, rate = res[rank]
        assert slowest == 2.0                      # max over ranks, seen by every rank
        assert rate == pytest.approx(world * 100.0 / 2e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(10.0, 1, 2.0) == pytest.approx(5000.0)
