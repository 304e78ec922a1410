"""The multi-rank timing of bench.py on CPU: two gloo ranks, no GPU.

The step shards over nothing (one GPU computes a whole layer), so bench.py --gpus N runs N
independent replicas.  Each rank times its own steps; the job is as slow as its slowest
rank, so the reported time is the max over ranks and the throughput counts every rank's
tokens.
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


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], "cpu", world)
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    times = [6.5, 7.25]
    mp.start_processes(_rank, args=(2, port, times, out), nprocs=2, join=True, start_method="spawn")
    assert dict(out) == {0: 7.25, 1: 7.25}


def test_single_rank_and_throughput():
    assert bench.max_over_ranks(3.0, "cpu", 1) == 3.0
    # 16384 tokens per replica and step, 2 replicas, 6.4 ms per step
    assert bench.job_tokens_per_second(16384, 2, 6.4) == pytest.approx(2 * 16384 / 6.4e-3)
