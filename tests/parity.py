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


def _kept_set_valid(s, got, c, budget):
    """True when ``got`` (the engine's ascending candidate ids, ``budget`` of
    them) is a top-``budget`` set of ``s`` up to the near-tie band: every kept
    score is >= the budget-th largest minus the band and every dropped one <=
    it plus the band.  The same test as the set comparison in
    :func:`check_unit`, without sorting all c scores."""
    sb = -np.partition(-s, budget - 1)[budget - 1]
    band = SEL_BAND * np.max(np.abs(s))
    kept = np.zeros(c, bool)
    kept[got] = True
    ok = s[kept].min() >= sb - band
    if c > budget:
        ok = ok and s[~kept].max() <= sb + band
    return ok


def check_all_units(batch: Batch, group, w, budget, lambdas, mode, threads=8,
                    block_tokens=1 << 22):
    """Every unit of ``batch`` against the oracle: one engine score call in
    ``mode``, then select + compact for each lambda.  a, r, m of every
    candidate within the tolerance (window rows exactly 0); the kept set of
    every unit and lambda valid up to the tie band, ascending, the window
    after it, -1 past nk; K'/V' bit-exact gathers of the engine's own indices
    (checked on the device).  The oracle (importance and the O(N d) closed
    form of the row mean) runs unit by unit on ``threads`` host threads."""
    from concurrent.futures import ThreadPoolExecutor
    if mode == "gemm_sym":
        eng = Engine(group, w, max_units=batch.num_units, max_tokens=batch.num_tokens,
                     redundancy="gemm", symmetric_gemm=True)
    else:
        eng = Engine(group, w, max_units=batch.num_units, max_tokens=batch.num_tokens,
                     redundancy=mode)
    U = batch.num_units
    off = batch.tok_off_host
    a, r = eng.alloc_scores(batch)
    m = torch.full_like(a, float("nan"))
    eng.score(batch, a, r, m)
    eng.check_status()
    ah, rh, mh = (t.cpu().numpy() for t in (a, r, m))
    del m
    idx_h, nk_h = [], []
    off_dev = torch.from_numpy(off[:-1].astype(np.int64)).to(batch.K.device)
    for lam in lambdas:
        idx, nk, Ko, Vo = eng.alloc_outputs(batch, budget)
        eng.select(batch, a, r, lam, budget, idx, nk)
        eng.compact(batch, idx, nk, budget, Ko, Vo)
        eng.check_status()
        # compaction, on the device, in blocks of units
        ub = max(1, (1 << 28) // (Ko.shape[1] * 256))
        for u0 in range(0, U, ub):
            u1 = min(U, u0 + ub)
            ib = idx[u0:u1].long()
            valid = ib >= 0
            assert torch.equal(valid.sum(1).int(), nk[u0:u1]), "nk disagrees with the -1 fill"
            src = (ib + off_dev[u0:u1, None]).clamp(min=0)
            for X, Xo in ((batch.K, Ko), (batch.V, Vo)):
                want = X[src].view(torch.int16)
                want[~valid] = 0
                assert torch.equal(Xo[u0:u1].view(torch.int16), want), \
                    f"lambda {lam}: compaction differs in units {u0}..{u1 - 1}"
        idx_h.append(idx.cpu().numpy())
        nk_h.append(nk.cpu().numpy())
        del idx, nk, Ko, Vo
    del a, r
    eng.close()
    torch.cuda.empty_cache()
    Qh = batch.Q.double().cpu().numpy()

    def one(u, k):
        N = k.shape[0]
        c = N - w
        lo = int(off[u])
        _, a_o = ora.importance(Qh[u], k)
        m_o, r_o = ora.redundancy_mean_closed_form(k, w)
        close(ah[lo:lo + c], a_o, f"unit {u} a")
        close(rh[lo:lo + c], r_o, f"unit {u} r")
        close(mh[lo:lo + c], m_o, f"unit {u} m")
        assert np.all(ah[lo + c:lo + N] == 0) and np.all(rh[lo + c:lo + N] == 0), \
            f"unit {u}: window rows must be 0"
        for li, lam in enumerate(lambdas):
            nk = int(nk_h[li][u])
            got = idx_h[li][u]
            assert np.all(got[nk:] == -1), f"unit {u}: -1 fill"
            got = got[:nk]
            if c <= budget:
                assert np.array_equal(got, np.arange(N)), f"unit {u} lambda {lam}: keep all"
                continue
            assert nk == budget + w
            assert np.all(np.diff(got) > 0), f"unit {u} lambda {lam}: not ascending"
            assert np.array_equal(got[budget:], np.arange(c, N)), f"unit {u}: window"
            s = ora.joint_score(a_o, r_o, lam)
            assert _kept_set_valid(s, got[:budget], c, budget), \
                f"unit {u} lambda {lam}: kept set differs outside the tie band"
        return u

    with ThreadPoolExecutor(threads) as ex:
        u0 = 0
        while u0 < U:
            u1 = u0 + 1
            while u1 < U and off[u1 + 1] - off[u0] <= block_tokens:
                u1 += 1
            Kh = batch.K[int(off[u0]):int(off[u1])].cpu()   # one copy per block
            futs = [ex.submit(lambda u=u: one(u, Kh[int(off[u] - off[u0]):
                                                     int(off[u + 1] - off[u0])].double().numpy()))
                    for u in range(u0, u1)]
            for f in futs:
                f.result()
            u0 = u1
    return U
