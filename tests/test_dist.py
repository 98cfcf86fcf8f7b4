"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The op shards with no data-path exchange: each rank runs its own batch
(weak scaling). What needs ranks is the plumbing: distinct per-rank inputs,
the max-over-ranks timing reduction and the whole-job aggregate.
"""
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


def _worker(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.WORKLOADS["tiny"]
        seed = bench.rank_seed(w, rank)
        inp = workloads.make_inputs(w, seed=seed)
        mine = [1.0 + rank, 10.0 - rank, 5.0]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, (seed, float(inp.q.sum())))
        out[rank] = (got, gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    for rank in range(world):
        got, gathered = out[rank]
        assert got == [2.0, 10.0, 5.0]          # element-wise max over ranks
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world          # every rank draws its own batch
        assert gathered[0][1] != gathered[1][1]


def test_aggregate_is_whole_job():
    import bench
    assert bench.aggregate_tokens_per_s(4, 1000, 2.0) == pytest.approx(2_000_000.0)
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
