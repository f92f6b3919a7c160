"""Splitting one batch of units across GPUs.

Units (sequence, layer, KV head) are independent, so a multi-GPU run needs no
exchange on the data path: each rank compresses a subset of the units.  The
subsets are balanced by a per-unit cost (greedy longest-processing-time-first
assignment).  With the redundancy GEMM the step is dominated by the N x N tile
products, so a unit of N tokens costs about N^2 + 320 N (the linear term is the
HBM-bound scoring and selection: 128 N^2 tensor flops at ~1 PFLOP/s against
about 264 N bytes at ~6.5 TB/s break even near N = 320); with the closed-form
redundancy every step is HBM-bound and a unit costs N.
"""
from __future__ import annotations

import heapq
from typing import List

import numpy as np


def unit_cost(n_tokens, redundancy: str = "gemm") -> np.ndarray:
    """Relative cost of compressing units of the given lengths."""
    n = np.asarray(n_tokens, dtype=np.float64)
    if redundancy == "closed":
        return n
    if redundancy in ("gemm", "max"):
        return n * (n + 320.0)
    raise ValueError(redundancy)


def shard_units(n_tokens, world: int, redundancy: str = "gemm") -> List[np.ndarray]:
    """Assign unit indices to `world` ranks, balancing the summed unit cost
    (:func:`unit_cost`) per rank.

    Costliest unit first, each to the currently least-loaded rank (ties to the
    lower rank).  Returns, per rank, its unit indices in ascending order."""
    n = np.asarray(n_tokens, dtype=np.int64)
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = unit_cost(n, redundancy)
    order = np.lexsort((np.arange(len(n)), -cost))   # cost descending, index ascending
    heap = [(0.0, r) for r in range(world)]
    parts = [[] for _ in range(world)]
    for u in order.tolist():
        load, r = heapq.heappop(heap)
        parts[r].append(u)
        heapq.heappush(heap, (load + float(cost[u]), r))
    return [np.array(sorted(p), dtype=np.int64) for p in parts]


def sub_offsets(tok_off, units) -> np.ndarray:
    """Row offsets of the sub-batch made of `units` (in the given order)."""
    off = np.asarray(tok_off, dtype=np.int64)
    n = off[np.asarray(units, dtype=np.int64) + 1] - off[np.asarray(units, dtype=np.int64)]
    out = np.zeros(len(n) + 1, dtype=np.int64)
    np.cumsum(n, out=out[1:])
    return out


def gather_rows(tok_off, units) -> np.ndarray:
    """Global K/V row indices of the sub-batch, unit after unit."""
    off = np.asarray(tok_off, dtype=np.int64)
    if len(units) == 0:
        return np.zeros(0, dtype=np.int64)
    return np.concatenate([np.arange(off[u], off[u + 1]) for u in units])
