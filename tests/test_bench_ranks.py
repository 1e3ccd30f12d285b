"""The replica timing of bench.py on several ranks, without a GPU: two gloo
processes on the CPU take the max over ranks and the whole-job rate the way
the benchmark does under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank               # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, device="cpu")
        out[rank] = (ms_max, bench.job_rate(100, world, ms_max))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_on_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms_max, rate = out[r]
        assert ms_max == 15.0                # every rank sees the slowest time
        assert rate == pytest.approx(world * 100 / 0.015)


def test_job_rate_single_rank():
    import bench
    assert bench.job_rate(4000, 1, 80.0) == pytest.approx(50_000.0)
