"""Host-side logic of the multi-GPU path.

Users are independent: no attention crosses users and M-FALCON candidates
touch only their own user, so a batch shards by user with no collective on
the data path.  ``lpt_partition`` splits users across ranks by longest
processing time first on an estimated cost; ``shard_offsets`` builds one
rank's jagged batch; ``reduce_timing`` combines per-rank timings the way the
bench reports them (time = max over ranks, work = sum over ranks).
"""
from __future__ import annotations

import heapq
from typing import List, Sequence, Tuple

import numpy as np


def user_cost(lengths: Sequence[int], d_model: int, n_heads: int, d_qk: int, d_v: int) -> np.ndarray:
    """Estimated forward cost per user: projections (linear in n) plus causal
    attention (quadratic in n), in flops."""
    n = np.asarray(lengths, np.float64)
    F = 2 * n_heads * (d_qk + d_v)
    proj = n * (2.0 * d_model * F + 2.0 * n_heads * d_v * d_model)
    attn = n_heads * (2.0 * d_qk + 2.0 * d_v) * n * (n + 1) / 2.0
    return proj + attn


def lpt_partition(costs: Sequence[float], world: int) -> List[List[int]]:
    """Assign items to `world` bins, largest cost first, each to the currently
    lightest bin (ties: lowest rank).  Returns sorted item lists per rank."""
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = np.asarray(costs, np.float64)
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap: List[Tuple[float, int]] = [(0.0, r) for r in range(world)]
    bins: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        bins[r].append(i)
        heapq.heappush(heap, (load + float(costs[i]), r))
    return [sorted(b) for b in bins]


def shard_offsets(offsets: Sequence[int], users: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """Offsets of the sub-batch made of `users` (in the given order) and the
    row indices of the full batch that it gathers."""
    offsets = np.asarray(offsets, np.int64)
    lens = np.array([offsets[u + 1] - offsets[u] for u in users], dtype=np.int64)
    sub = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    rows = (np.concatenate([np.arange(offsets[u], offsets[u + 1]) for u in users])
            if len(users) else np.zeros(0, np.int64))
    return sub, rows.astype(np.int64)


def reduce_timing(ms: float, units: float, group=None) -> Tuple[float, float]:
    """(max over ranks of ms, sum over ranks of units) through torch.distributed
    (any backend); without an initialised group, the local values."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(ms), float(units)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend(group) == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    u = torch.tensor([units], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(u, op=dist.ReduceOp.SUM, group=group)
    return float(t.item()), float(u.item())
