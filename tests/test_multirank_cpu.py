"""Multi-process path of bench.py on CPU: two gloo ranks (no GPU).

The bench shards work by heads (weak scaling): each rank runs the whole workload on its
own heads, the job time is the slowest rank's and the executed pairs add up.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from free_block_sparse_plan_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, pairs = bench.reduce_over_ranks(10.0 + rank, 1000.0 * (rank + 1), world, "cpu")
        w = bench.rank_workload(W.TINY, rank, world)
        Q, _, _ = W.make_head(w, 0)
        out[rank] = (ms, pairs, float(Q[0, 0]), w.seed)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_max_and_pairs_sum():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, pairs, _, _ = res[r]
        assert ms == 11.0                    # slowest rank
        assert pairs == 3000.0               # 1000 + 2000
    # every rank draws its own heads
    assert res[0][3] != res[1][3] and res[0][2] != res[1][2]


def test_single_rank_is_identity():
    assert bench.reduce_over_ranks(3.5, 42.0, 1, "cpu") == (3.5, 42.0)
    assert bench.rank_workload(W.TINY, 0, 1) is W.TINY
