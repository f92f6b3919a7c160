"""Pure-Python loop transcription of the same definitions, for tiny inputs.

TEST INFRASTRUCTURE (only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` may use it).  It is a second, independent
transcription of the R-KV steps (R-KV article, "R-KV三步走": 重要性打分,
冗余打分, 联合淘汰) written with scalar ``math`` only -- no NumPy -- so that a
slip in the vectorised oracle (a transposed operand, a wrong axis, a missing
mask) shows up as a disagreement.  Inputs are nested lists of floats.
"""
from __future__ import annotations

import itertools
import math


def _dot(x, y):
    return math.fsum(a * b for a, b in zip(x, y))


def importance(Q, K):
    """Q[g][t] (d floats), K[j] (d floats) -> (a_bar over all N, a over C)."""
    G, w, N, d = len(Q), len(Q[0]), len(K), len(K[0])
    abar = [0.0] * N
    for g in range(G):
        for t in range(w):
            last = N - w + t                        # causal: keys 0..last
            z = [_dot(Q[g][t], K[j]) / math.sqrt(d) for j in range(last + 1)]
            zmax = max(z)
            e = [math.exp(v - zmax) for v in z]
            tot = math.fsum(e)
            for j in range(last + 1):
                abar[j] += e[j] / tot / (G * w)
    c = N - w
    tot = math.fsum(abar[:c])
    return abar, [abar[i] / tot for i in range(c)]


def redundancy(K, w):
    """Row mean of the cosine-similarity matrix, diagonal excluded, then a
    softmax over the candidates."""
    N = len(K)
    c = N - w
    unit = []
    for k in K:
        n = math.sqrt(_dot(k, k))
        unit.append([x / n for x in k] if n > 0 else [0.0] * len(k))
    m = []
    for i in range(c):
        acc = math.fsum(_dot(unit[i], unit[j]) for j in range(N) if j != i)
        m.append(acc / (N - 1))
    mx = max(m)
    e = [math.exp(v - mx) for v in m]
    tot = math.fsum(e)
    return m, [v / tot for v in e]


def redundancy_max(K, w):
    """Row max of the cosine-similarity matrix, diagonal excluded, then a
    softmax over the candidates."""
    N = len(K)
    c = N - w
    unit = []
    for k in K:
        n = math.sqrt(_dot(k, k))
        unit.append([x / n for x in k] if n > 0 else [0.0] * len(k))
    m = [max(_dot(unit[i], unit[j]) for j in range(N) if j != i) for i in range(c)]
    mx = max(m)
    e = [math.exp(v - mx) for v in m]
    tot = math.fsum(e)
    return m, [v / tot for v in e]


def select(s, N, w, budget):
    """Sort candidates by (score descending, index ascending)."""
    c = N - w
    if c <= budget:
        return list(range(N))
    order = sorted(range(c), key=lambda i: (-s[i], i))
    return sorted(order[:budget]) + list(range(c, N))


def select_by_subsets(s, N, w, budget):
    """Brute force over every budget-subset of the candidates: the kept set
    maximises the total score; among equal totals the lexicographically
    smallest sorted index list wins.  Only for N <= ~14."""
    c = N - w
    if c <= budget:
        return list(range(N))
    best, best_val = None, None
    for sub in itertools.combinations(range(c), budget):
        val = math.fsum(s[i] for i in sub)
        if best_val is None or val > best_val + 1e-15:
            best, best_val = list(sub), val
    return best + list(range(c, N))


def run_unit(Q, K, w, budget, lam):
    N = len(K)
    abar, a = importance(Q, K)
    m, r = redundancy(K, w)
    s = [lam * ai - (1.0 - lam) * ri for ai, ri in zip(a, r)]
    return dict(abar=abar, a=a, m=m, r=r, s=s, idx=select(s, N, w, budget))


def evict_in_place(N, idx):
    """Live-slot mask and ascending free slots, by a plain scan."""
    kept = set(int(i) for i in idx)
    keep = [i in kept for i in range(N)]
    free = [i for i in range(N) if not keep[i]]
    return keep, free


def refree_keep_count(p, sinks, T):
    """Stopping rule by a plain loop over the ranking (sinks, then newest first)."""
    N = len(p)
    m = min(sinks, N)
    order = list(range(m)) + list(range(N - 1, m - 1, -1))
    total = math.fsum(x * x for x in p)
    acc = 0.0
    for k, j in enumerate(order, start=1):
        acc += p[j] * p[j]
        if math.sqrt(acc) >= (1.0 - T) * math.sqrt(total):
            return k
    return N
