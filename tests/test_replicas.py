"""The multi-GPU bench path on the CPU: two gloo ranks stand in for two GPUs.

The decode path shards by sequence with no exchange step, so N GPUs run N
independent replicas; the ranks meet only to agree on the slowest rank's time.
These tests run that host logic (rank environment, per-rank seeds, max over ranks,
whole-job throughput) in two processes over gloo on 127.0.0.1.
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


def _rank_main(rank, world, port, elapsed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.replica_env()
        dist.barrier()
        slowest = bench.max_over_ranks(elapsed[rank], w)
        job_bytes = bench.sum_over_ranks(1_000_000 * (1 + rank), w)   # replicas differ
        value = bench.job_throughput(job_bytes, 10, slowest)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.replica_seed(7, r))
        out[rank] = (w, r, lr, slowest, value, tuple(seeds))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_agree_on_the_slowest_rank():
    world, port = 2, _free_port()
    elapsed = [3.0, 5.0]   # ms: rank 1 is slower
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, elapsed, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        w, r, lr, slowest, value, seeds = res[rank]
        assert (w, r, lr) == (2, rank, rank)
        assert slowest == 5.0                      # max over ranks, on every rank
        # (1 + 2) MB per step x 10 steps over 5 ms = 6 GB/s
        assert value == pytest.approx(6.0)
        assert seeds == (7, 8)                     # distinct replicas


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.sum_over_ranks(4.0, 1) == 4.0
    assert bench.job_throughput(2_000_000_000, 3, 1000.0) == pytest.approx(6.0)
