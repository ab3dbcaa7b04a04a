"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): each rank
runs the same workload, the job time is the maximum over ranks and the rate
counts every rank's work.  The kernels are not involved: the path has no
data-path collective (replicas of independent problems)."""
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


def _rank_main(rank, world, port, times_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(times_ms[rank], True, device="cpu")
        out[rank] = t
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_job_time_is_max_over_ranks(world):
    times = [3.0, 7.5][:world]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, out), nprocs=world, join=True,
                       start_method="spawn")
    assert [out[r] for r in range(world)] == [max(times)] * world


def test_job_throughput_counts_every_rank():
    # 2 ranks x 1e12 flop per step x 10 steps in 20 ms (slowest rank) = 1e15 flop/s
    assert bench.job_throughput(2, 1e12, 10, 20.0) == pytest.approx(1e15)
    assert bench.job_throughput(1, 1e12, 10, 20.0) == pytest.approx(5e14)


def test_single_rank_needs_no_group():
    assert bench.max_over_ranks(4.2, False) == 4.2
