"""The multi-GPU path of bench.py runs independent replicas (no data-path collective):
the only cross-rank steps are a barrier and the max-over-ranks reduction of the timed
region.  Exercised here with two gloo ranks on the CPU."""

import os
import socket

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
        bench.barrier(world, device="cpu")
        # rank r "took" 10 + 5 r ms: the job time is the slowest rank's
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world, device="cpu")
        out[rank] = t
        bench.barrier(world, device="cpu")
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_replica_throughput_is_whole_job():
    # 2 replicas x 16 sequences x 50 steps in 400 ms (slowest rank) = 4000 tokens/s
    assert bench.replica_tokens_per_s(2, 16, 50, 400.0) == 4000.0
    assert bench.replica_tokens_per_s(1, 16, 50, 400.0) == 2000.0
