"""The benchmark's multi-rank host logic on CPU with gloo, world size 2: the
step time is the max over ranks, the value counts every rank's units, and the
reference arm runs on rank 0 only."""
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
        ms = 100.0 + 50.0 * rank                      # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms)
        value = bench.aggregate_throughput(1000, world, 10, ms_max)
        out[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1]
    ms_max, value = out[0]
    assert ms_max == 150.0
    assert value == pytest.approx(1000 * 2 * 10 / 0.150)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5) == 3.5


def test_reference_arm_other_ranks_exit_without_work():
    class A:
        workload = "tiny_fp32"
        steps = 1
        warmup = 3
        reference_budget_s = 1.0
    assert bench.run_reference(A, rank=1, world=2) == 0
