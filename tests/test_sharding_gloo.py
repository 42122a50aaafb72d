"""Multi-rank host logic on CPU (gloo, world size 2): user sharding covers
every user exactly once and balances the estimated cost; the bench's
reduction takes the max time and the summed work over ranks; a sharded batch
gives each rank exactly its users' rows (checked with the oracle on CPU)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import hstu_workloads as hw
from hstu_sequential_transducer_layer_b200 import sharding as S


def test_lpt_partition_properties():
    rng = np.random.default_rng(0)
    costs = rng.lognormal(0, 1.5, size=200)
    for world in (1, 2, 3, 8):
        bins = S.lpt_partition(costs, world)
        allu = sorted(u for b in bins for u in b)
        assert allu == list(range(200))
        loads = [costs[b].sum() for b in bins]
        # LPT bound: max load <= mean load + largest item
        assert max(loads) <= np.mean(loads) + costs.max() + 1e-9


def test_shard_offsets_rows():
    off = np.array([0, 3, 3, 10, 12])
    sub, rows = S.shard_offsets(off, [2, 0])
    assert sub.tolist() == [0, 7, 10]
    assert rows.tolist() == [3, 4, 5, 6, 7, 8, 9, 0, 1, 2]


def test_user_cost_monotone():
    c = S.user_cost([1, 10, 100], 64, 2, 32, 32)
    assert c[0] < c[1] < c[2]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from oracle import hstu_oracle as O
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dims = hw.LayerDims(32, 2, 16, 8, 32, 32, 2, 0, 1e-6, hw.FP32)
        w = hw.custom("shard", [5, 9, 1, 14, 3, 7], dims, seed=3)
        costs = S.user_cost(w.lengths, 32, 2, 16, 8)
        mine = S.lpt_partition(costs, world)[rank]
        sub, rows = S.shard_offsets(w.offsets, mine)
        y = O.layer_fwd(w.X[rows], sub, w.timestamps[rows], w.weights[0], dims)
        full = O.layer_fwd(w.X, w.offsets, w.timestamps, w.weights[0], dims)
        ok = bool(np.allclose(y, full[rows], rtol=0, atol=1e-12))
        ms, units = S.reduce_timing(float(10 + rank), float(len(rows)))
        objs = [None] * world
        dist.all_gather_object(objs, mine)
        q.put((rank, ok, ms, units, objs))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, ms, units, objs in res:
        assert ok
        assert ms == 11.0                  # max over ranks
        assert units == 5 + 9 + 1 + 14 + 3 + 7   # every row exactly once
        cover = sorted(u for b in objs for u in b)
        assert cover == list(range(6))
