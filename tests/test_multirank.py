"""Multi-rank host logic on CPU (gloo, world size 2): shards are distinct and
independent, and timings reduce to the slowest rank.  No GPU is involved."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from selective_state_space_32_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.WORKLOADS["tiny_f32"]
        g = W.generate(w.B, w.L, w.D, w.N, w.dtype, w.h0_std, w.reset_frac,
                       seed=bench.shard_seed(w, rank))
        # each rank times its own shard; the job's time is the slowest rank's
        mine = [10.0 + rank, 5.0 - rank]
        got = bench.max_over_ranks(mine, world)
        # shards differ: gather a checksum of each rank's u
        cs = torch.tensor([float(np.abs(g["u"]).sum())], dtype=torch.float64)
        allcs = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allcs, cs)
        out[rank] = (got, [float(c) for c in allcs])
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        got, cs = out[r]
        assert got == [11.0, 5.0]
        assert cs[0] != cs[1]


def test_single_rank_reduce_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
