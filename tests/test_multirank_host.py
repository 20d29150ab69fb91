"""The benchmark's multi-rank host logic on CPU ranks (gloo, world size 2): replicas are
weak-scaled, the job time is the slowest rank's (max over ranks, seen by every rank), and
the job rate counts every rank's units against that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own_ms = 2.0 + rank * 1.5                    # rank 1 is the slow one
        bench.barrier(world)
        job_ms = bench.max_over_ranks(own_ms, world, device="cpu")
        rate = bench.job_throughput(1000.0, world, job_ms)
        out[rank] = torch.tensor([own_ms, job_ms, rate], dtype=torch.float64)
    finally:
        dist.destroy_process_group()


def test_two_rank_job_time_is_the_slowest_rank():
    world = 2
    out = torch.zeros(world, 3, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[:, 1].tolist() == [3.5, 3.5]          # both ranks see the max
    assert out[0, 2].item() == pytest.approx(1000.0 * 2 / 3.5e-3)


def test_single_rank_is_unchanged():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(4.25, 1) == 4.25
    assert bench.job_throughput(500.0, 1, 2.0) == pytest.approx(250000.0)
