"""The benchmark's multi-rank host logic on CPU: two gloo ranks, the job time
is the slowest rank's and the throughput counts every rank's batch."""

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
        ms = bench.max_over_ranks(10.0 + 5.0 * rank)   # rank 1 is slower
        out[rank] = ms
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_job_throughput_counts_all_ranks():
    # 8x1024x768 channel-steps per rank, 10 steps, 2 ranks, 1 ms
    v = bench.job_throughput(8 * 1024 * 768, 10, 2, 1.0)
    assert v == pytest.approx(2 * 8 * 1024 * 768 * 10 / 1e-3 / 1e9)
