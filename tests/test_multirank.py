"""The N > 1 path of bench.py on CPU: two gloo ranks, each running its own
replica of the workload (no data-path collective), time = max over ranks, and
the reported value aggregates the work of all ranks."""
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
        # each rank "measures" a different time; the job time is the slowest rank
        mine = 10.0 + 5.0 * rank
        out[rank] = bench.max_over_ranks(mine, world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_aggregate_is_whole_job_throughput():
    # 2 ranks x 3 steps x 1e12 FLOP in 1.5 s (slowest rank) = 4 TFLOP/s
    assert bench.aggregate_tflops(1e12, 3, 1500.0, 2) == pytest.approx(4.0)
    assert bench.max_over_ranks(7.0, 1) == 7.0


def test_reference_arm_other_ranks_exit_without_work():
    class A:
        steps, warmup = 1, 1
    assert bench.run_reference(A(), rank=1, world=2) == 0
