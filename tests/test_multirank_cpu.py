"""The benchmark's multi-rank host logic with two gloo ranks on CPU: each rank
gates its own token shard (no collective on the data path), the reported time
is the slowest rank's, and throughput counts every rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        slowest = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        wl = bench.rank_workload(workloads.TINY, rank)
        first_row = wl.hidden_rows(0, 1)
        out[rank] = (slowest, bench.job_tokens_per_s(world, wl.T, 100, slowest), wl.seed, first_row.tobytes())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:  # no fork of this (multi-threaded) process
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0            # both ranks report the slowest rank's time
    assert res[0][1] == pytest.approx(2 * 64 * 100 / 0.015)
    assert res[0][2] != res[1][2]                    # different token shards
    assert res[0][3] != res[1][3]


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5
    assert bench.job_tokens_per_s(1, 1000, 10, 1000.0) == 10000.0
    assert bench.rank_workload(workloads.TRAIN, 0) == workloads.TRAIN
