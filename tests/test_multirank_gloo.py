"""Multi-GPU plumbing of the benchmark, exercised on CPU with two gloo ranks.

The hot path shards by request only (replicas, no data-path collective); the one
cross-rank step is the max-over-ranks timing reduction and the barrier around the
timed region.  These run here on gloo over 127.0.0.1; on GPUs the same code runs
over NCCL.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world)
        value = bench.replica_throughput(3.0e12, slowest, world)
        out[rank] = (slowest, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_slowest_step_and_whole_job_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    slowest, value = res[0]
    assert slowest == 15.0
    assert value == pytest.approx(2 * 3.0e12 / 15e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.replica_throughput(1.0e12, 10.0, 1) == pytest.approx(1.0e14)
