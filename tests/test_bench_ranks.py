"""Host logic of the multi-GPU bench on CPU: two gloo ranks (processes) reduce their step
times to the slowest one and compute the whole-job throughput the same way; only rank 0
reports.  No GPU: each rank plays one GPU's part with made-up step times."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.5 if rank == 0 else 2.5                   # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, world)
        value = bench.job_tflops(3.0e12, world, worst)
        dist.barrier()
        out[rank] = (worst, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step_time():
    world = 2
    out = mp.Manager().dict()
    mp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1]
    worst, value = out[0]
    assert worst == 2.5
    assert value == pytest.approx(2 * 3.0e12 / 2.5e-3 / 1e12)    # 2400 TFLOP/s for the job


def test_single_rank_is_a_no_op():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_tflops(2.0e12, 1, 1.0) == pytest.approx(2000.0)
