"""Replica timing across ranks (gloo, world size 2, CPU).

With --gpus N every rank runs its own replica of the step and no collective
touches the data path; the whole-job number divides the units all ranks
processed by the slowest rank's time. These tests run that aggregation on two
CPU processes.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    import datetime

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        out[rank] = (ms, bench.replica_gbs(1e9, 10, world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world, port = 2, _free_port()
    times = [3.0, 7.5]  # rank 1 is the slow replica
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, times, out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ms, gbs = out[r]
        assert ms == pytest.approx(7.5)
        # 2 replicas x 10 steps x 1 GB in 7.5 ms
        assert gbs == pytest.approx(2 * 10 * 1e9 / 7.5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(4.25) == 4.25
    assert bench.replica_gbs(2e9, 5, 1, 10.0) == pytest.approx(1000.0)
