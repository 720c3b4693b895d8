"""Multi-GPU runs are replicas: every rank decodes its own sequence and the only
collectives are the timing barrier and the max over ranks. This checks that host
logic with world_size 2 on the gloo backend (CPU processes, 127.0.0.1)."""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out) -> None:
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "took" 100 + 50 r ms for 10 steps: the job is timed by the slowest
        ms = bench.max_over_ranks(100.0 + 50.0 * rank, world, "cpu")
        dist.barrier()
        out[rank] = (ms, bench.replica_rate(10, world, ms / 1e3))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_rate_gloo_world2():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        ms, rate = res[rank]
        assert ms == 150.0                       # the slowest rank, on every rank
        assert rate == pytest.approx(2 * 10 / 0.150)  # all ranks' units over the slowest time


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.replica_rate(100, 1, 2.0) == 50.0
