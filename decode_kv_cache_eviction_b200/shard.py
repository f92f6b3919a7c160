"""Splitting one batch of units across GPUs.

Units (sequence, layer, KV head) are independent, so a multi-GPU run needs no
exchange on the data path: each rank compresses a subset of the units.  The
subsets are balanced by token count (greedy longest-first assignment), which
balances both the HBM-bound scoring (proportional to N) and, nearly, the
redundancy GEMM (proportional to N^2) for ragged batches.
"""
from __future__ import annotations

import heapq
from typing import List

import numpy as np


def shard_units(n_tokens, world: int) -> List[np.ndarray]:
    """Assign unit indices to `world` ranks, balancing the sum of N per rank.

    Longest unit first, each to the currently least-loaded rank (ties to the
    lower rank).  Returns, per rank, its unit indices in ascending order."""
    n = np.asarray(n_tokens, dtype=np.int64)
    if world < 1:
        raise ValueError("world must be >= 1")
    order = np.lexsort((np.arange(len(n)), -n))      # N descending, index ascending
    heap = [(0, r) for r in range(world)]
    parts = [[] for _ in range(world)]
    for u in order.tolist():
        load, r = heapq.heappop(heap)
        parts[r].append(u)
        heapq.heappush(heap, (load + int(n[u]), r))
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
