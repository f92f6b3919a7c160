"""Helpers for comparing the CUDA engine with the fp64 oracle.

Tolerances (written here once, used by every parity test):
* a, r, m: |x_gpu - x_oracle| <= 1e-6 + 1e-3 * |x_oracle| elementwise over the
  candidates; window rows must be exactly 0.
* kept indices: identical sets, except tokens whose oracle joint score lies
  within 1e-5 * max_i |s_i| of the budget-th largest score (a near tie that
  fp32 scoring may legitimately order either way).
* select alone (given the same fp32 a and r): bit-exact, with the ranking
  decided in fp32 on both sides.
* compaction: bit-exact rows.
"""
from __future__ import annotations

import numpy as np
import torch

from decode_kv_cache_eviction_b200 import Batch, Engine
from decode_kv_cache_eviction_b200 import workloads as W
from oracle import rkv_oracle as ora

ATOL, RTOL = 1e-6, 1e-3
SEL_BAND = 1e-5


def rand_batch(lengths, G, w, seed=0, dup=0.2, zero_rows=(), device="cuda:0"):
    """Gaussian keys, values and queries for units of the given lengths; a
    fraction ``dup`` of each unit's rows are exact copies of earlier rows."""
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    K = rng.standard_normal((T, 128)).astype(np.float32)
    for u in range(len(lengths)):
        for i in range(1, lengths[u]):
            if rng.random() < dup:
                K[off[u] + i] = K[off[u] + rng.integers(0, i)]
    for z in zero_rows:
        K[z] = 0
    V = rng.standard_normal((T, 128)).astype(np.float32)
    Q = rng.standard_normal((len(lengths), G, w, 128)).astype(np.float32)
    t = lambda x: torch.from_numpy(x).to(device).to(torch.bfloat16)
    return Batch(t(K), t(V), t(Q), off)


def make_batch(gen_batch: W.Batch) -> Batch:
    return Batch(gen_batch.K, gen_batch.V, gen_batch.Q, gen_batch.tok_off)


def run_engine(batch: Batch, group, window, lam, budget, mode="gemm", single_cta=False,
               engine=None, symmetric=False):
    """Score, select and compact with a fresh engine (mode "gemm_sym" = the
    symmetric row-mean GEMM)."""
    if mode == "gemm_sym":
        mode, symmetric = "gemm", True
    eng = engine or Engine(group, window, max_units=max(1, batch.num_units),
                           max_tokens=max(1, batch.num_tokens), redundancy=mode,
                           single_cta_gemm=single_cta, symmetric_gemm=symmetric)
    a, r = eng.alloc_scores(batch)
    m = torch.full_like(a, float("nan"))
    a.fill_(float("nan"))
    r.fill_(float("nan"))
    eng.score(batch, a, r, m)
    idx, nk, Ko, Vo = eng.alloc_outputs(batch, budget)
    eng.select(batch, a, r, lam, budget, idx, nk)
    eng.compact(batch, idx, nk, budget, Ko, Vo)
    eng.check_status()
    torch.cuda.synchronize()
    return dict(a=a.cpu().numpy(), r=r.cpu().numpy(), m=m.cpu().numpy(),
                idx=idx.cpu().numpy(), nk=nk.cpu().numpy(), Ko=Ko, Vo=Vo, engine=eng)


def unit_inputs(batch: Batch, u: int):
    """fp64 copies of unit u's K, V, Q (exact widening of the bf16 bytes)."""
    r0, r1 = int(batch.tok_off_host[u]), int(batch.tok_off_host[u + 1])
    k = batch.K[r0:r1].float().cpu().numpy().astype(np.float64)
    v = batch.V[r0:r1].float().cpu().numpy().astype(np.float64)
    q = batch.Q[u].float().cpu().numpy().astype(np.float64)
    return k, v, q


def close(x_gpu, x_ora, what):
    x_gpu = np.asarray(x_gpu, dtype=np.float64)
    err = np.abs(x_gpu - x_ora)
    lim = ATOL + RTOL * np.abs(x_ora)
    bad = np.nonzero(~(err <= lim))[0]
    assert bad.size == 0, (f"{what}: {bad.size} of {x_ora.size} out of tolerance; first "
                           f"{bad[:5].tolist()} gpu={x_gpu[bad[:5]].tolist()} "
                           f"oracle={x_ora[bad[:5]].tolist()}")


def oracle_mode(mode):
    """The oracle redundancy that an engine mode computes."""
    return "max" if mode == "max" else "closed"   # gemm, gemm_sym, closed: the row mean


def check_unit(out, batch: Batch, u, w, lam, budget, redundancy="closed", check_m=True):
    """Compare unit u of an engine run with the oracle.  ``redundancy`` names the
    oracle function: ``closed`` / ``rowblocks`` (row mean) or ``max`` (row max)."""
    k, v, q = unit_inputs(batch, u)
    N = k.shape[0]
    c = N - w
    r0 = int(batch.tok_off_host[u])
    _, a_o = ora.importance(q, k)
    if redundancy == "closed":
        m_o, r_o = ora.redundancy_mean_closed_form(k, w)
    elif redundancy == "max":
        m_o, r_o = ora.redundancy_max(k, w)
    else:
        m_o, r_o = ora.redundancy_mean(k, w)
    a_g = out["a"][r0:r0 + N]
    r_g = out["r"][r0:r0 + N]
    close(a_g[:c], a_o, f"unit {u} a")
    close(r_g[:c], r_o, f"unit {u} r")
    assert np.all(a_g[c:] == 0) and np.all(r_g[c:] == 0), "window rows must be 0"
    if check_m:
        close(out["m"][r0:r0 + c], m_o, f"unit {u} m")
    # kept set vs the oracle, with the near-tie band
    s_o = ora.joint_score(a_o, r_o, lam)
    want = ora.select(s_o, N, w, budget)
    nk = int(out["nk"][u])
    got = out["idx"][u, :nk]
    assert nk == len(want)
    assert np.all(np.diff(got) > 0), "kept indices must ascend"
    if c > budget:
        assert np.array_equal(got[budget:], np.arange(c, N))
        g_set, w_set = set(got[:budget].tolist()), set(want[:budget].tolist())
        diff = g_set ^ w_set
        if diff:
            sb = np.sort(s_o)[::-1][budget - 1]
            band = SEL_BAND * np.max(np.abs(s_o))
            far = [i for i in diff if abs(s_o[i] - sb) > band]
            assert not far, f"unit {u}: kept sets differ outside the tie band: {far[:5]}"
    else:
        assert np.array_equal(got, np.arange(N))
    assert np.all(out["idx"][u, nk:] == -1)
    # compaction is bit-exact given the engine's own indices
    Kc = out["Ko"][u].cpu()
    Vc = out["Vo"][u].cpu()
    src = torch.from_numpy(got.astype(np.int64)) + r0
    assert torch.equal(Kc[:nk].view(torch.int16), batch.K[src.to(batch.K.device)].cpu().view(torch.int16))
    assert torch.equal(Vc[:nk].view(torch.int16), batch.V[src.to(batch.K.device)].cpu().view(torch.int16))
    assert torch.count_nonzero(Kc[nk:].view(torch.int16)) == 0
    assert torch.count_nonzero(Vc[nk:].view(torch.int16)) == 0
    return dict(a=a_o, r=r_o, m=m_o, s=s_o)
