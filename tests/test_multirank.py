"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): every rank's time is
reduced with MAX, and the job throughput counts all ranks' steps over that time."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]
        got = bench.max_over_ranks(ms, world, torch.device("cpu"))
        out[rank] = (got, bench.job_throughput(1e12, 10, world, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        ms, tf = out[r]
        assert ms == 20.0                      # the slowest rank
        assert tf == pytest.approx(1e12 * 10 * 2 / 20e-3 / 1e12)


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    assert bench.job_throughput(2e12, 5, 1, 10.0) == pytest.approx(1000.0)
