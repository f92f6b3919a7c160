"""Seeded synthetic decode-shaped KV caches.

This module only draws random numbers and arranges them into the shapes and
duplicate structure of the five workloads below; it holds none of the scoring,
selection or compaction arithmetic.  Both the CUDA path and the fp64 oracle read
the bytes it produces.

A *unit* is one (sequence, layer, KV head).  Unit ``u`` owns the contiguous key
and value rows ``tok_off[u] .. tok_off[u+1]-1`` of ``K`` and ``V`` (``[T, d]``
bf16), and ``G * w`` window queries ``Q[u]`` (``[G, w, d]`` bf16, query head
``g`` of the group, window step ``t``).

Recipe (shared by every workload):

* Raw keys, values and queries are i.i.d. N(0, 1).
* A fraction of key positions is turned into copies of earlier keys: a copied
  position holds the raw key at the root of its copy chain (the chain always
  points backwards, so it ends at a position that is not a copy) plus fresh
  N(0, noise^2) noise (noise = 0 gives exact duplicates).
* Copies come either as single tokens (position uniform, source uniform among
  earlier positions) or as non-overlapping spans (destination spans spread by
  random gaps, each source span drawn uniformly among spans that end before the
  destination starts).
* Optional per-(unit, channel) key scale drawn U(lo, hi), applied after copying.
* Everything is rounded to bf16 (round to nearest even).

The duplicate layout is drawn with NumPy PCG64 seeded from (seed, workload,
unit) so it does not depend on the device; the Gaussian values come from a
torch generator on the requested device (CPU for small oracle-only cases, CUDA
for full-size caches).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic decode-cache batch."""

    name: str
    n_seq: int                  # sequences in the batch
    n_layer: int                # layers per sequence
    n_kv_head: int              # KV heads per layer
    group: int                  # G: query heads per KV head
    head_dim: int               # d
    window: int                 # w: window queries (and always-kept tail keys)
    budget: int                 # B: kept candidates per unit
    lambdas: tuple              # joint-score weights to run
    n_min: int                  # per-sequence token count drawn U[n_min, n_max]
    n_max: int
    dup_frac: float             # fraction of key positions that are copies
    dup_noise: float            # std of the noise added to a copy
    span_len: Optional[tuple]   # (lo, hi) span length; None = single-token copies
    key_scale: Optional[tuple]  # (lo, hi) per-(unit, channel) scale; None = none

    @property
    def num_units(self) -> int:
        return self.n_seq * self.n_layer * self.n_kv_head


# The five decode-cache workloads; index i is the i-th configuration of the
# scope table (tiny, one Llama-3-8B layer, a full R1-Llama-8B cache, a 32K
# reasoning trace, a ragged serving batch).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 1, 128, 8, 256, (0.1,), 1024, 1024,
                     0.20, 0.05, None, None),
    "llama3_8b_layer": Workload("llama3_8b_layer", 1, 1, 8, 4, 128, 8, 1024,
                                (0.1,), 4096, 4096, 0.25, 0.05, (64, 64),
                                (0.5, 4.0)),
    "r1_llama8b_cache": Workload("r1_llama8b_cache", 8, 32, 8, 4, 128, 8, 2048,
                                 (0.1,), 16384, 16384, 0.25, 0.05, (64, 64),
                                 None),
    "long_trace_32k": Workload("long_trace_32k", 4, 32, 8, 4, 128, 8, 4096,
                               (0.1,), 32768, 32768, 0.30, 0.05, (32, 256),
                               None),
    "ragged_serving": Workload("ragged_serving", 64, 32, 8, 4, 128, 8, 1024,
                               (0.0, 0.1, 1.0), 2048, 8192, 0.15, 0.0, None,
                               None),
}
WORKLOAD_ORDER = ["tiny", "llama3_8b_layer", "r1_llama8b_cache",
                  "long_trace_32k", "ragged_serving"]

# The R1-Llama-8B cache at its trigger cadence: compression runs every 128
# decode steps, when the cache holds the B = 2048 kept tokens plus 128 new
# ones (N = 2176).  CADENCE gives (decode steps per trigger, trace length).
WORKLOADS["r1_llama8b_cadence"] = Workload("r1_llama8b_cadence", 8, 32, 8, 4, 128, 8, 2048,
                                           (0.1,), 2176, 2176, 0.25, 0.05, (64, 64), None)
CADENCE = {"r1_llama8b_cadence": (128, 16384)}
EXTRA_WORKLOADS = ["r1_llama8b_cadence"]


def custom(name="custom", n_seq=1, n_layer=1, n_kv_head=1, group=1, head_dim=128,
           window=8, budget=64, lambdas=(0.1,), n_min=512, n_max=None,
           dup_frac=0.2, dup_noise=0.05, span_len=None, key_scale=None):
    """A small workload with the same recipe (for tests)."""
    return Workload(name, n_seq, n_layer, n_kv_head, group, head_dim, window,
                    budget, tuple(lambdas), n_min,
                    n_min if n_max is None else n_max, dup_frac, dup_noise,
                    span_len, key_scale)


def _rng(seed: int, *keys: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *keys])))


def _name_key(name: str) -> int:
    return int.from_bytes(name.encode()[:8].ljust(8, b"\0"), "little") & 0x7FFFFFFF


def seq_lengths(wl: Workload, seed: int) -> np.ndarray:
    """Per-sequence cached-token counts (all units of a sequence share N)."""
    if wl.n_min == wl.n_max:
        return np.full(wl.n_seq, wl.n_min, dtype=np.int64)
    rng = _rng(seed, _name_key(wl.name), 0x5E9)
    return rng.integers(wl.n_min, wl.n_max + 1, size=wl.n_seq).astype(np.int64)


def unit_lengths(wl: Workload, seed: int) -> np.ndarray:
    per_seq = seq_lengths(wl, seed)
    return np.repeat(per_seq, wl.n_layer * wl.n_kv_head)


def token_offsets(wl: Workload, seed: int) -> np.ndarray:
    n = unit_lengths(wl, seed)
    off = np.zeros(len(n) + 1, dtype=np.int64)
    np.cumsum(n, out=off[1:])
    return off


def _copy_sources(wl: Workload, n: int, rng: np.random.Generator) -> np.ndarray:
    """src[i] = i for an original position, else an earlier position."""
    src = np.arange(n, dtype=np.int64)
    n_copy = int(round(wl.dup_frac * n))
    if n_copy == 0 or n < 2:
        return src
    if wl.span_len is None:
        pos = rng.choice(np.arange(1, n), size=min(n_copy, n - 1), replace=False)
        src[pos] = (rng.random(len(pos)) * pos).astype(np.int64)
    else:
        lo, hi = wl.span_len
        lens = []
        total = 0
        while total < n_copy:
            ln = int(rng.integers(lo, hi + 1))
            lens.append(ln)
            total += ln
        lens = np.array(lens, dtype=np.int64)
        lead = hi                        # room for a source before the first span
        free = n - lead - int(lens.sum())
        if free < 0:                     # cache too short for the requested spans
            keep = np.cumsum(lens) <= max(n - lead, 0)
            lens = lens[keep]
            free = n - lead - int(lens.sum())
        if len(lens) == 0:
            return src
        cuts = np.sort(rng.integers(0, free + 1, size=len(lens)))
        gaps = np.diff(np.concatenate([[0], cuts]))
        starts = lead + np.cumsum(gaps) + np.concatenate([[0], np.cumsum(lens)[:-1]])
        for st, ln in zip(starts.tolist(), lens.tolist()):
            s0 = int(rng.integers(0, st - ln + 1))
            src[st:st + ln] = np.arange(s0, s0 + ln)
    # pointer jumping: every chain points backwards, so this reaches the roots
    while True:
        nxt = src[src]
        if np.array_equal(nxt, src):
            break
        src = nxt
    return src


def copy_maps(wl: Workload, seed: int, units: Optional[Sequence[int]] = None):
    """Per-unit copy-source maps (unit-local positions)."""
    n = unit_lengths(wl, seed)
    units = range(wl.num_units) if units is None else units
    return {u: _copy_sources(wl, int(n[u]), _rng(seed, _name_key(wl.name), 1 + u))
            for u in units}


def _gen(device, seed: int, tag: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + tag) & 0x7FFFFFFFFFFFFFFF)
    return g


@dataclasses.dataclass
class Batch:
    """One generated batch: bf16 tensors on ``device`` plus host offsets."""

    workload: Workload
    seed: int
    K: torch.Tensor          # [T, d] bf16
    V: torch.Tensor          # [T, d] bf16
    Q: torch.Tensor          # [U, G, w, d] bf16
    tok_off: np.ndarray      # [U+1] int64 (host)
    tok_off_dev: torch.Tensor  # [U+1] int64 on device

    @property
    def num_units(self):
        return len(self.tok_off) - 1

    @property
    def n_tokens(self):
        return np.diff(self.tok_off)


def generate(wl: Workload, seed: int = 0, device="cpu",
             units_per_chunk: int = 256) -> Batch:
    """Generate the whole batch of ``wl`` on ``device``."""
    device = torch.device(device)
    d = wl.head_dim
    off = token_offsets(wl, seed)
    T = int(off[-1])
    U = wl.num_units
    K = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    V = torch.empty((T, d), dtype=torch.bfloat16, device=device)
    gk, gv, gq, gn, gs = (_gen(device, seed, t) for t in (11, 12, 13, 14, 15))
    for u0 in range(0, U, units_per_chunk):
        u1 = min(U, u0 + units_per_chunk)
        r0, r1 = int(off[u0]), int(off[u1])
        raw = torch.randn((r1 - r0, d), generator=gk, device=device)
        maps = copy_maps(wl, seed, range(u0, u1))
        src = np.concatenate([maps[u] + (off[u] - r0) for u in range(u0, u1)])
        is_copy = src != np.arange(r1 - r0)
        src_t = torch.from_numpy(src).to(device)
        keys = raw[src_t]
        if wl.dup_noise > 0 and is_copy.any():
            noise = torch.randn((r1 - r0, d), generator=gn, device=device)
            mask = torch.from_numpy(is_copy).to(device)
            keys = torch.where(mask[:, None], keys + wl.dup_noise * noise, keys)
        if wl.key_scale is not None:
            lo, hi = wl.key_scale
            sc = lo + (hi - lo) * torch.rand((u1 - u0, d), generator=gs, device=device)
            lens = torch.from_numpy(np.diff(off[u0:u1 + 1])).to(device)
            keys = keys * torch.repeat_interleave(sc, lens, dim=0)
        K[r0:r1] = keys.to(torch.bfloat16)
        del raw, keys
        V[r0:r1] = torch.randn((r1 - r0, d), generator=gv, device=device).to(torch.bfloat16)
    Q = torch.randn((U, wl.group, wl.window, d), generator=gq,
                    device=device).to(torch.bfloat16)
    return Batch(wl, seed, K, V, Q, off, torch.from_numpy(off).to(device))


def unit_host_arrays(batch: Batch, u: int):
    """Unit ``u``'s K, V [N, d] and Q [G, w, d] as float64 NumPy arrays
    (exact widening of the bf16 values)."""
    r0, r1 = int(batch.tok_off[u]), int(batch.tok_off[u + 1])
    k = batch.K[r0:r1].float().cpu().numpy().astype(np.float64)
    v = batch.V[r0:r1].float().cpu().numpy().astype(np.float64)
    q = batch.Q[u].float().cpu().numpy().astype(np.float64)
    return k, v, q
