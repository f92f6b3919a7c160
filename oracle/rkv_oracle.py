"""fp64 CPU oracle for decode-time KV-cache scoring, selection and compaction.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import or run anything in this directory.  The
product path (the CUDA library and its Python binding) never calls it and shares
no code with it.

Source: the R-KV article (QbitAI repost, "R-KV三步走：冗余识别+重要性评估+动态淘汰"),
which names the method's steps in this order:

* 边生成边压缩 (decoding-time compression): the step runs on the cache of one
  (sequence, layer, KV head) while decoding;
* 重要性打分 (importance): multi-head attention estimates each token's
  contribution to what follows;
* 冗余打分 (redundancy): cosine similarity between key vectors finds repeated
  content;
* 联合淘汰 (joint eviction): keep high-importance, low-redundancy tokens within
  the KV budget, best at lambda ~ 0.1.

The page gives only these ingredients.  The exact formulas written out below
are the reading this engine adopts for them (plain attention softmax averaged
over window queries and the GQA group; row-mean cosine similarity with the
diagonal excluded, then a softmax over tokens; s = lam*a - (1-lam)*r; keep the
last w tokens and the top-B of the rest, ties to the lower index).

Notation: one unit has N cached keys K [N, d] (and values V), window w, group G,
queries Q [G, w, d]; query (g, t) sits at position N - w + t and attends to keys
j <= N - w + t.  Candidates C = {0 .. N-w-1}.  Everything is float64; inputs
are the exact widening of the bf16 values.
"""
from __future__ import annotations

import numpy as np


def key_norms(K: np.ndarray) -> np.ndarray:
    """||k_i|| for every key (冗余打分 needs cosine similarity, i.e. unit keys)."""
    return np.sqrt(np.einsum("nd,nd->n", K, K))


def unit_keys(K: np.ndarray) -> np.ndarray:
    """k_hat_i = k_i / ||k_i||, with k_hat_i = 0 for a zero key."""
    nrm = key_norms(K)
    inv = np.zeros_like(nrm)
    nz = nrm > 0
    inv[nz] = 1.0 / nrm[nz]
    return K * inv[:, None]


def attention_probs(Q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """p[g, t, j]: causal softmax of q_{g,t} . k_j / sqrt(d) over j <= N-w+t
    (重要性打分: the attention that the most recent decode queries pay to each
    cached token).  Masked entries are exactly 0."""
    G, w, d = Q.shape
    N = K.shape[0]
    # every logit q_{g,t} . k_j at once: one [G*w, d] x [d, N] matrix product
    z = (Q.reshape(G * w, d) @ K.T).reshape(G, w, N) / np.sqrt(d)
    pos = N - w + np.arange(w)                       # position of query t
    visible = np.arange(N)[None, :] <= pos[:, None]  # [w, N]
    z = np.where(visible[None], z, -np.inf)
    zmax = z.max(axis=2, keepdims=True)
    e = np.exp(z - zmax)
    return e / e.sum(axis=2, keepdims=True)


def importance(Q: np.ndarray, K: np.ndarray):
    """Importance (重要性打分).

    a_bar_j = mean over (g, t) of p[g, t, j]; a_i = a_bar_i / sum_{j in C} a_bar_j
    for i in C.  Returns (a_bar [N], a [N - w])."""
    G, w, d = Q.shape
    N = K.shape[0]
    abar = attention_probs(Q, K).mean(axis=(0, 1))
    c = N - w
    if c <= 0:
        return abar, np.zeros(0)
    return abar, abar[:c] / abar[:c].sum()


def redundancy_mean(K: np.ndarray, w: int, block: int = 2048):
    """Redundancy (冗余打分), straight from the definition, in row blocks.

    S_ij = k_hat_i . k_hat_j; m_i = sum_{j != i, j < N} S_ij / (N - 1) for i in C;
    r = softmax over C of m.  The N x N matrix is never held whole.
    Returns (m [N - w], r [N - w])."""
    N = K.shape[0]
    c = N - w
    if c <= 0:
        return np.zeros(0), np.zeros(0)
    kh = unit_keys(K)
    m = np.empty(c)
    for i0 in range(0, c, block):
        i1 = min(c, i0 + block)
        S = kh[i0:i1] @ kh.T                              # [rows, N]
        S[np.arange(i1 - i0), np.arange(i0, i1)] = 0.0    # exclude j == i
        m[i0:i1] = S.sum(axis=1) / (N - 1)
    return m, softmax(m)


def redundancy_mean_closed_form(K: np.ndarray, w: int):
    """The same m as :func:`redundancy_mean`, by linearity of the row sum:
    sum_{j != i} k_hat_i . k_hat_j = k_hat_i . U - k_hat_i . k_hat_i with
    U = sum_j k_hat_j.  O(N d) instead of O(N^2 d); exact up to rounding."""
    N = K.shape[0]
    c = N - w
    if c <= 0:
        return np.zeros(0), np.zeros(0)
    kh = unit_keys(K)
    U = kh.sum(axis=0)
    m = (kh[:c] @ U - np.einsum("nd,nd->n", kh[:c], kh[:c])) / (N - 1)
    return m, softmax(m)


def redundancy_max(K: np.ndarray, w: int, block: int = 2048):
    """Redundancy as the nearest duplicate (冗余打分, row-max reading): the
    largest cosine similarity to any other cached key,
    m_i = max_{j != i, j < N} k_hat_i . k_hat_j for i in C; r = softmax over C.
    A key with an exact copy elsewhere gets m = 1, the largest possible value.
    Returns (m [N - w], r [N - w])."""
    N = K.shape[0]
    c = N - w
    if c <= 0:
        return np.zeros(0), np.zeros(0)
    kh = unit_keys(K)
    m = np.empty(c)
    for i0 in range(0, c, block):
        i1 = min(c, i0 + block)
        S = kh[i0:i1] @ kh.T
        S[np.arange(i1 - i0), np.arange(i0, i1)] = -np.inf   # exclude j == i
        m[i0:i1] = S.max(axis=1)
    return m, softmax(m)


def softmax(x: np.ndarray) -> np.ndarray:
    if x.size == 0:
        return x.copy()
    e = np.exp(x - x.max())
    return e / e.sum()


def joint_score(a: np.ndarray, r: np.ndarray, lam: float) -> np.ndarray:
    """Joint eviction score (联合淘汰): s_i = lam * a_i - (1 - lam) * r_i."""
    return lam * a - (1.0 - lam) * r


def select(s: np.ndarray, N: int, w: int, budget: int):
    """Kept indices (联合淘汰 under the KV budget).

    Rank candidates by (s descending, index ascending); keep the first
    min(budget, N - w); return them in ascending order followed by the window
    N - w .. N - 1.  If N - w <= budget every token is kept."""
    c = N - w
    if c <= budget:
        return np.arange(N, dtype=np.int64)
    order = np.lexsort((np.arange(c), -s))     # primary key: -s; then index
    kept = np.sort(order[:budget])
    return np.concatenate([kept, np.arange(c, N)]).astype(np.int64)


def select_with_sinks(s: np.ndarray, N: int, w: int, budget: int, sinks: int):
    """Kept indices with attention-sink protection and a per-unit budget (the
    ReFreeKV review keeps the first m tokens as anchors; LU-KV gives each head
    its own budget).  The first min(sinks, N - w) tokens are always kept, the
    top-`budget` of the remaining candidates sinks .. N-w-1 are ranked by (s
    descending, index ascending) as in :func:`select`, and the window follows.
    Returns sinks, then the selected candidates ascending, then the window;
    every token when no more than `budget` candidates remain.  With sinks = 0
    this is :func:`select`."""
    c = N - w
    m = min(sinks, c)
    if c - m <= budget:
        return np.arange(N, dtype=np.int64)
    rest = s[m:c]
    order = np.lexsort((np.arange(c - m), -rest))
    kept = np.sort(order[:budget]) + m
    return np.concatenate([np.arange(m), kept, np.arange(c, N)]).astype(np.int64)


def last_query_probs(Q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """The attention row of the newest query (ReFreeKV with k = 1: one row of
    the attention matrix stands for all of it), averaged over the GQA group:
    p_j = mean_g softmax_j(q_{g, w-1} . k_j / sqrt(d)), over all N keys."""
    return attention_probs(Q, K)[:, -1, :].mean(axis=0)


def refree_keep_count(p: np.ndarray, sinks: int, T: float) -> int:
    """ReFreeKV's stopping rule on one attention row p [N].

    Initial ranking: the first m = min(sinks, N) tokens in order, then the
    others from the newest to the oldest.  Uni-Metric: the Frobenius norm of
    the attention entries kept, which the review calls their energy.  Cutting
    stops once the energy lost, the drop of that norm from the full row's, is
    at most T of it: the smallest k with ||p_first k|| >= (1 - T) ||p||, i.e.
    sum_{first k} p^2 >= (1 - T)^2 sum p^2."""
    N = len(p)
    m = min(sinks, N)
    order = np.concatenate([np.arange(m), np.arange(N - 1, m - 1, -1)])
    e = p[order] ** 2
    need = (1.0 - T) ** 2 * e.sum()
    kept = np.cumsum(e)
    return int(np.argmax(kept >= need)) + 1


def refree_budget(k: int, N: int, w: int, sinks: int) -> int:
    """The R-KV budget that keeps k tokens in all: k minus the sinks and the
    window (which are kept anyway), at least 0."""
    c = N - w
    return max(0, k - min(sinks, c) - w)


def compact(K: np.ndarray, V: np.ndarray, idx: np.ndarray):
    """Gather-based compaction of the surviving rows (the R-KV-style baseline
    named in the ThinKV summary): K'[j] = K[idx[j]], V'[j] = V[idx[j]]."""
    return K[idx], V[idx]


def evict_in_place(N: int, idx: np.ndarray):
    """In-place slot reuse (the ThinKV summary's Continuous Thinking: evicted
    slots are not compacted away but reused).  Given the kept token indices of
    a unit, returns (keep [N] bool, free [N - kept] int64): the live-slot mask
    and the evicted slots in ascending order, which new tokens take next."""
    keep = np.zeros(N, dtype=bool)
    keep[np.asarray(idx, dtype=np.int64)] = True
    free = np.flatnonzero(~keep).astype(np.int64)
    return keep, free


def fill_free_slots(K: np.ndarray, V: np.ndarray, keep: np.ndarray, free: np.ndarray,
                    K_new: np.ndarray, V_new: np.ndarray):
    """New tokens overwrite evicted slots (Continuous Thinking): new token t goes
    to slot free[t], lowest slot first; the slot becomes live.  Returns the
    updated (K, V, keep); the inputs are not modified.  Needs len(K_new) <=
    len(free)."""
    n = len(K_new)
    assert n <= len(free) and len(V_new) == n
    K2, V2, keep2 = K.copy(), V.copy(), keep.copy()
    slots = np.asarray(free[:n], dtype=np.int64)
    K2[slots] = K_new
    V2[slots] = V_new
    keep2[slots] = True
    return K2, V2, keep2


def run_unit(Q, K, V, w: int, budget: int, lam: float, redundancy="rowblocks"):
    """Whole path for one unit.  ``redundancy`` picks the row-mean definition
    (``rowblocks``), its closed form (``closed``) or the row-max reading
    (``max``)."""
    N = K.shape[0]
    abar, a = importance(Q, K)
    if redundancy == "rowblocks":
        m, r = redundancy_mean(K, w)
    elif redundancy == "closed":
        m, r = redundancy_mean_closed_form(K, w)
    elif redundancy == "max":
        m, r = redundancy_max(K, w)
    else:
        raise ValueError(redundancy)
    s = joint_score(a, r, lam)
    idx = select(s, N, w, budget)
    Kc, Vc = compact(K, V, idx)
    return dict(abar=abar, a=a, m=m, r=r, s=s, idx=idx, K=Kc, V=Vc,
                norms=key_norms(K))
