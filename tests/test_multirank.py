"""Rank plumbing of the replicas-only multi-GPU bench, on CPU with gloo (world size 2).

Sequence-heads are independent, so ranks exchange nothing on the data path: each rank
draws its own copy of the workload (rank-specific seed) and only the timing is reduced
(max over ranks)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workload


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank, world)
        wl, mode = bench.rank_workload("gdn2_t4k", rank)
        small = workload.Workload("s", B=1, H=1, T=8, dk=16, dv=16, chunk=16, dtype="f32",
                                  mode=wl.mode, seed=wl.seed, s0_std=0.1)
        q = workload.make_inputs(small)["q"]
        g = [torch.zeros_like(q) for _ in range(world)]
        dist.all_gather(g, q)
        lo, hi = workload.shard_range(10, rank, world)
        out[rank] = dict(t=t, seed=wl.seed, differs=not torch.equal(g[0], g[1]), lo=lo, hi=hi)
    finally:
        dist.destroy_process_group()


def test_replicas_reduce_only_timing():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    assert r0["t"] == r1["t"] == 2.5            # max over ranks
    assert r0["seed"] != r1["seed"]             # each rank its own workload copy
    assert r0["differs"] and r1["differs"]
    assert (r0["lo"], r0["hi"], r1["lo"], r1["hi"]) == (0, 5, 5, 10)


def test_shard_range_covers_units_exactly():
    for n in (0, 1, 7, 128, 129):
        for world in (1, 2, 3, 8):
            parts = [workload.shard_range(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            for (a, b), (c, d) in zip(parts, parts[1:]):
                assert b == c and b >= a
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
