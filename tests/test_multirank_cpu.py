"""The N > 1 host path of bench.py on CPU: two ranks over gloo.

The path shards by sequence with no exchange step, so N GPUs run N replicas;
what is shared between ranks is only the whole-job arithmetic (longest time
over ranks, bytes of all ranks) and the rule that gives every rank its own
sequences. Both run here with world_size 2 on the gloo backend.
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


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), ".."))
    import bench
    import workloads as wk
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        t, b = bench.over_ranks(10.0 + 5.0 * rank, 1000 * (rank + 1), world, "cpu")
        wl = bench.rank_workload(wk.get("tiny"), rank, world)
        keep = wk.prefill_inputs(wl, 0)["keep"]
        seeds = [None] * world
        dist.all_gather_object(seeds, (wl.seed, keep.sum().item()))
        out[rank] = (t, b, seeds)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in range(2):
        t, b, seeds = res[rank]
        assert t == 15.0                      # the longest time over ranks
        assert b == 3000.0                    # bytes of both ranks
        assert seeds[0][0] != seeds[1][0]     # each rank its own sequences
        assert seeds[0][1] != seeds[1][1]


def test_single_rank_is_local():
    import bench
    import workloads as wk
    assert bench.over_ranks(12.5, 77, 1, "cpu") == (12.5, 77.0)
    wl = wk.get("tiny")
    assert bench.rank_workload(wl, 0, 1) is wl
