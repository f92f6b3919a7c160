"""GPU engine vs the fp64 oracle, through the C ABI (see tests/parity.py for the
tolerances).  Ordered from the integer kernels (select, compaction) to the
score kernels, then edge cases, then the full-size workloads on sampled units and on every unit."""
import json
import os

import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Batch, Engine, RkvError
from decode_kv_cache_eviction_b200 import workloads as W
from oracle import rkv_oracle as ora

from parity import (check_all_units, check_unit, make_batch, oracle_mode, rand_batch, run_engine,
                    unit_inputs)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


# ----------------------------------------------------------------- select alone
@pytest.mark.parametrize("lam", [0.0, 0.1, 1.0])
@pytest.mark.parametrize("lengths,budget", [([1000], 100), ([4096, 300, 9], 256),
                                            ([20000, 33000], 4096), ([5000], 0),
                                            ([65536, 131072], 4096)])
def test_select_bit_exact_given_scores(lam, lengths, budget):
    w = 8
    b = rand_batch(lengths, 1, w, seed=len(lengths) + budget)
    rng = np.random.default_rng(budget)
    T = b.num_tokens
    a = rng.random(T).astype(np.float32) * 1e-3
    r = rng.random(T).astype(np.float32) * 1e-3
    a[::7] = a[3]  # plenty of exact ties
    r[::7] = r[3]
    eng = Engine(1, w, max_units=len(lengths), max_tokens=T, redundancy="closed")
    ta, tr = torch.from_numpy(a).to(DEV), torch.from_numpy(r).to(DEV)
    idx, nk, _, _ = eng.alloc_outputs(b, budget)
    eng.select(b, ta, tr, lam, budget, idx, nk)
    eng.check_status()
    idx, nk = idx.cpu().numpy(), nk.cpu().numpy()
    lam32 = np.float32(lam)
    for u, N in enumerate(lengths):
        r0 = int(b.tok_off_host[u])
        c = N - w
        s32 = ora.joint_score(a[r0:r0 + c], r[r0:r0 + c], lam32)   # fp32 on both sides
        assert s32.dtype == np.float32
        want = ora.select(s32, N, w, budget)
        assert nk[u] == len(want)
        np.testing.assert_array_equal(idx[u, :nk[u]], want)
        assert np.all(idx[u, nk[u]:] == -1)


@pytest.mark.parametrize("nan_frac", [0.1, 0.95])
def test_select_nan_and_signed_zero_scores(nan_frac):
    """A NaN score ranks below every number and -0 ties with +0 (index order),
    as in the oracle's ranking; with most scores NaN the bracket cannot hold the
    budget's rank and the selection runs over all candidates."""
    w, budget = 8, 700
    lengths = [5000, 3001, 700 + w + 5]
    b = rand_batch(lengths, 1, w, seed=11)
    rng = np.random.default_rng(12)
    T = b.num_tokens
    a = (rng.random(T).astype(np.float32) - 0.5) * 1e-3
    r = rng.random(T).astype(np.float32) * 1e-3
    a[rng.random(T) < nan_frac] = np.nan
    z = rng.random(T) < 0.05           # exact zeros of either sign: s = +-0
    a[z] = np.where(rng.random(z.sum()) < 0.5, np.float32(-0.0), np.float32(0.0))
    r[z] = 0.0
    eng = Engine(1, w, max_units=len(lengths), max_tokens=T, redundancy="closed")
    ta, tr = torch.from_numpy(a).to(DEV), torch.from_numpy(r).to(DEV)
    idx, nk, _, _ = eng.alloc_outputs(b, budget)
    eng.select(b, ta, tr, 0.3, budget, idx, nk)
    eng.check_status()
    idx, nk = idx.cpu().numpy(), nk.cpu().numpy()
    for u, N in enumerate(lengths):
        r0 = int(b.tok_off_host[u])
        c = N - w
        s32 = ora.joint_score(a[r0:r0 + c], r[r0:r0 + c], np.float32(0.3))
        want = ora.select(s32, N, w, budget)
        assert nk[u] == len(want)
        np.testing.assert_array_equal(idx[u, :nk[u]], want)


@pytest.mark.parametrize("n,budget", [(40000, 1000), (3000, 2999), (9000, 1)])
def test_select_all_scores_equal(n, budget):
    """Every score ties: the bracket around the budget's rank holds every
    candidate, so the selection runs over all of them; ties go to the lowest
    indices."""
    w = 8
    b = rand_batch([n], 1, w, seed=9)
    a = torch.full((n,), 2e-4, dtype=torch.float32, device=DEV)
    r = torch.full((n,), 1e-4, dtype=torch.float32, device=DEV)
    eng = Engine(1, w, max_units=1, max_tokens=n, redundancy="closed")
    idx, nk, _, _ = eng.alloc_outputs(b, budget)
    eng.select(b, a, r, 0.1, budget, idx, nk)
    eng.check_status()
    got = idx[0, :nk[0]].cpu().numpy()
    want = np.arange(n) if n - w <= budget else np.concatenate([np.arange(budget),
                                                                np.arange(n - w, n)])
    np.testing.assert_array_equal(got, want)


def test_select_two_clusters_and_outliers():
    """Scores in two tight clusters plus a few extreme outliers (the sample
    still brackets the budget's rank, or the full selection takes over)."""
    w, n, budget = 8, 50000, 7000
    rng = np.random.default_rng(5)
    a = np.where(rng.random(n) < 0.8, 1e-5 + 1e-9 * rng.random(n), 3e-5 + 1e-9 * rng.random(n))
    a[rng.choice(n, 20, replace=False)] = 0.5
    a = a.astype(np.float32)
    r = np.full(n, 1e-5, np.float32)
    b = rand_batch([n], 1, w, seed=10)
    eng = Engine(1, w, max_units=1, max_tokens=n, redundancy="closed")
    idx, nk, _, _ = eng.alloc_outputs(b, budget)
    for lam in (1.0, 0.3):
        eng.select(b, torch.from_numpy(a).to(DEV), torch.from_numpy(r).to(DEV), lam, budget,
                   idx, nk)
        eng.check_status()
        s32 = ora.joint_score(a[:n - w], r[:n - w], np.float32(lam))
        np.testing.assert_array_equal(idx[0, :nk[0]].cpu().numpy(), ora.select(s32, n, w, budget))


# ----------------------------------------------------------------- compaction alone
def test_compact_bit_exact_and_bad_index_flag():
    lengths, w, budget = [700, 64, 1500], 4, 100
    b = rand_batch(lengths, 1, w, seed=3)
    eng = Engine(1, w, max_units=3, max_tokens=b.num_tokens, redundancy="closed")
    U, Wd = 3, budget + w
    rng = np.random.default_rng(0)
    idx = np.full((U, Wd), -1, np.int32)
    nk = np.array([Wd, 64, 77], np.int32)
    for u, N in enumerate(lengths):
        idx[u, :nk[u]] = np.sort(rng.choice(N, size=nk[u], replace=False))
    tidx, tnk = torch.from_numpy(idx).to(DEV), torch.from_numpy(nk).to(DEV)
    _, _, Ko, Vo = eng.alloc_outputs(b, budget)
    eng.compact(b, tidx, tnk, budget, Ko, Vo)
    eng.check_status()
    for u in range(U):
        src = torch.from_numpy(idx[u, :nk[u]].astype(np.int64) + b.tok_off_host[u]).to(DEV)
        assert torch.equal(Ko[u, :nk[u]].view(torch.int16), b.K[src].view(torch.int16))
        assert torch.equal(Vo[u, :nk[u]].view(torch.int16), b.V[src].view(torch.int16))
        assert torch.count_nonzero(Ko[u, nk[u]:].view(torch.int16)) == 0
    # an index outside its unit zero-fills the row and is reported
    idx[1, 5] = 64
    tidx = torch.from_numpy(idx).to(DEV)
    eng.compact(b, tidx, tnk, budget, Ko, Vo)
    with pytest.raises(RkvError) as ei:
        eng.check_status()
    assert ei.value.code == -7
    assert torch.count_nonzero(Ko[1, 5].view(torch.int16)) == 0
    eng.check_status()   # the status word was cleared


# ----------------------------------------------------------------- worked example
def test_worked_example_on_gpu():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_6token.json")))
    K = np.zeros((6, 128), np.float32)
    K[:, :2] = np.array(g["K"])
    Q = np.zeros((1, 1, 2, 128), np.float32)
    Q[0, 0, :, :2] = np.array(g["Q"][0])
    # zero padding keeps every dot product and norm, but the kernel scales
    # logits by 1/sqrt(128) instead of 1/sqrt(2): pre-scale the queries by
    # sqrt(128/2) = 8 (exact in bf16) so the logits match the d = 2 example
    Q *= 8.0
    t = lambda x: torch.from_numpy(x).to(DEV).to(torch.bfloat16)
    b = Batch(t(K), t(K), t(Q), np.array([0, 6]))
    for mode in ("closed", "gemm", "gemm_sym"):
        for lam, want in g["idx"].items():
            out = run_engine(b, 1, 2, float(lam), 2, mode=mode)
            np.testing.assert_allclose(out["a"][:4], g["a"], atol=5e-6)
            np.testing.assert_allclose(out["r"][:4], g["r"], atol=5e-6)
            np.testing.assert_allclose(out["m"][:4], g["m"], atol=5e-6)
            assert out["idx"][0].tolist() == want, (mode, lam)
    # row max: nearest other unit key of each candidate, 1, 1, 1/sqrt(2), 0
    out = run_engine(b, 1, 2, 0.1, 2, mode="max")
    np.testing.assert_allclose(out["m"][:4], [1.0, 1.0, 0.5 ** 0.5, 0.0], atol=5e-6)
    np.testing.assert_allclose(out["a"][:4], g["a"], atol=5e-6)


# ----------------------------------------------------------------- score kernels, small
@pytest.mark.parametrize("mode", ["closed", "gemm", "max", "gemm_sym"])
@pytest.mark.parametrize("G,w", [(1, 8), (4, 8), (2, 3), (5, 5), (1, 1), (32, 1),
                                 # more than 32 query rows: one pass of 64 rows, or
                                 # several passes over row groups of 64
                                 (8, 8), (9, 7), (16, 5), (32, 8)])
def test_score_small_ragged(mode, G, w):
    lengths = [w, w + 1, 127, 128, 129, 1000, 2500, 5000]
    zero_rows = [3 + lengths[0] + lengths[1]]   # a zero key inside unit 2
    b = rand_batch(lengths, G, w, seed=G * 10 + w, zero_rows=zero_rows)
    budget = 64
    for lam in (0.1,):
        out = run_engine(b, G, w, lam, budget, mode=mode)
        for u in range(len(lengths)):
            check_unit(out, b, u, w, lam, budget, redundancy=oracle_mode(mode))


@pytest.mark.parametrize("G,w", [(4, 8), (8, 8)])   # one row group, then two
def test_intermediates_rho_and_U(G, w):
    """The score kernel's intermediates against their definitions: rho_j =
    1/||k_j|| (0 for a zero key), which the redundancy GEMM consumes, and the
    closed form's U = sum_j k_j/||k_j|| per unit."""
    lengths = [w, w + 1, 127, 1000, 5000, 33000]
    zero_rows = [3 + lengths[0] + lengths[1]]
    b = rand_batch(lengths, G, w, seed=G + 31, zero_rows=zero_rows)
    T, U = b.num_tokens, b.num_units
    for mode in ("gemm", "gemm_sym", "max"):
        eng = Engine(G, w, max_units=U, max_tokens=T,
                     redundancy="gemm" if mode == "gemm_sym" else mode,
                     symmetric_gemm=mode == "gemm_sym")
        a, r = eng.alloc_scores(b)
        eng.score(b, a, r)
        rho = torch.full((T,), float("nan"), device=DEV)
        eng.debug_intermediates(b, rho=rho)
        eng.check_status()
        with pytest.raises(RkvError):
            eng.debug_intermediates(b, U=torch.empty((U, 128), device=DEV))
        rho = rho.double().cpu().numpy()
        for u in range(U):
            k = unit_inputs(b, u)[0]
            nrm = ora.key_norms(k)
            want = np.where(nrm > 0, 1.0 / np.where(nrm > 0, nrm, 1.0), 0.0)
            lo, hi = int(b.tok_off_host[u]), int(b.tok_off_host[u + 1])
            np.testing.assert_allclose(rho[lo:hi], want, rtol=1e-5, atol=0, err_msg=f"{mode} unit {u}")
        eng.close()
    eng = Engine(G, w, max_units=U, max_tokens=T, redundancy="closed")
    a, r = eng.alloc_scores(b)
    eng.score(b, a, r)
    Ug = torch.full((U, 128), float("nan"), device=DEV)
    eng.debug_intermediates(b, U=Ug)
    eng.check_status()
    with pytest.raises(RkvError):
        eng.debug_intermediates(b, rho=torch.empty(T, device=DEV))
    Ug = Ug.double().cpu().numpy()
    for u in range(U):
        kh = ora.unit_keys(unit_inputs(b, u)[0])
        want = kh.sum(axis=0)
        # fp32 sums of N terms of magnitude <= 1: bound by the sum of magnitudes
        lim = 4e-5 * np.abs(kh).sum(axis=0) + 1e-6
        assert np.all(np.abs(Ug[u] - want) <= lim), (u, np.max(np.abs(Ug[u] - want) / lim))
    eng.close()


def test_row_max_flags_every_duplicate():
    """Row max: a candidate with an exact copy anywhere in its unit (window
    included) scores m = 1 up to fp32 rounding; the others stay well below."""
    lengths = [700, 3000, 129]
    b = rand_batch(lengths, 4, 8, seed=31, dup=0.25)
    out = run_engine(b, 4, 8, 0.1, 64, mode="max")
    K = b.K.float().cpu().numpy()
    for u, n in enumerate(lengths):
        r0 = int(b.tok_off_host[u])
        rows = K[r0:r0 + n]
        _, inv, cnt = np.unique(rows, axis=0, return_inverse=True, return_counts=True)
        has_copy = cnt[inv.reshape(-1)] > 1
        m = out["m"][r0:r0 + n - 8]
        assert np.all(np.abs(m[has_copy[:n - 8]] - 1.0) < 1e-5)
        assert np.all(m[~has_copy[:n - 8]] < 0.7)


@pytest.mark.parametrize("mode", ["closed", "gemm", "max", "gemm_sym"])
def test_budget_edges(mode):
    lengths = [300, 300, 300]
    w = 8
    b = rand_batch(lengths, 4, w, seed=7)
    for budget in (0, 1, 291, 292, 300):
        out = run_engine(b, 4, w, 0.1, budget, mode=mode)
        for u in range(3):
            check_unit(out, b, u, w, 0.1, budget, redundancy=oracle_mode(mode))


@pytest.mark.parametrize("mode", ["closed", "gemm", "max", "gemm_sym"])
def test_units_without_candidates(mode):
    """Units of exactly w tokens have no candidates: every token is kept, a and
    r are zero there, and the units around them are unaffected (the GEMM forms
    give such units no work items)."""
    w = 8
    lengths = [8, 300, 8, 9, 264, 8]
    b = rand_batch(lengths, 4, w, seed=23)
    out = run_engine(b, 4, w, 0.1, 16, mode=mode)
    for u in range(len(lengths)):
        check_unit(out, b, u, w, 0.1, 16, redundancy=oracle_mode(mode))


@pytest.mark.parametrize("mode", ["closed", "gemm_sym"])
def test_many_small_units(mode):
    """About 2000 short units in one batch (many score chunks, GEMM items and
    select CTAs of the short shape), checked on every 7th unit and on every
    unit's kept count."""
    w = 8
    rng = np.random.default_rng(37)
    lengths = rng.choice([8, 9, 16, 33, 100, 257, 300], size=2000).tolist()
    b = rand_batch(lengths, 4, w, seed=41, dup=0.1)
    out = run_engine(b, 4, w, 0.1, 12, mode=mode)
    for u in range(0, len(lengths), 7):
        check_unit(out, b, u, w, 0.1, 12, redundancy=oracle_mode(mode))
    want = [n if n - w <= 12 else 12 + w for n in lengths]
    assert out["nk"].tolist() == want


def test_unit_shorter_than_window_is_rejected():
    b = rand_batch([300, 5, 300], 4, 8, seed=29)
    eng = Engine(4, 8, max_units=3, max_tokens=b.num_tokens, redundancy="closed")
    a, r = eng.alloc_scores(b)
    with pytest.raises(RkvError) as e:
        eng.score(b, a, r)
    assert e.value.code == -1   # RKV_ERR_INVALID_ARG
    eng.close()


def test_gemm_single_cta_and_pair_agree():
    b = rand_batch([3000, 4100, 700], 4, 8, seed=11)
    o1 = run_engine(b, 4, 8, 0.1, 256, mode="gemm", single_cta=True)
    o2 = run_engine(b, 4, 8, 0.1, 256, mode="gemm", single_cta=False)
    o3 = run_engine(b, 4, 8, 0.1, 256, mode="closed")
    for u in range(3):
        check_unit(o1, b, u, 8, 0.1, 256)
    np.testing.assert_allclose(o1["m"], o2["m"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(o2["r"], o3["r"], rtol=1e-4, atol=1e-9)
    x1 = run_engine(b, 4, 8, 0.1, 256, mode="max", single_cta=True)
    x2 = run_engine(b, 4, 8, 0.1, 256, mode="max", single_cta=False)
    for u in range(3):
        check_unit(x1, b, u, 8, 0.1, 256, redundancy="max")
    # the same tile products and one max order per row: identical results
    assert np.array_equal(x1["m"], x2["m"])


@pytest.mark.parametrize("lengths", [[255, 256, 257, 511, 512, 513, 769], [3000, 4100, 700, 9],
                                     [20000, 12345],
                                     # last key block holds window tokens only
                                     [264, 520, 16, 1032, 258, 9]])
def test_symmetric_gemm_matches_dense(lengths):
    """Tiles on and above the diagonal only: the same m up to fp32 rounding
    order, the oracle's kept sets, and bit-identical repeated calls."""
    b = rand_batch(lengths, 4, 8, seed=len(lengths) * 13)
    dense = run_engine(b, 4, 8, 0.1, 128, mode="gemm")
    sym = run_engine(b, 4, 8, 0.1, 128, mode="gemm_sym")
    for u in range(len(lengths)):
        check_unit(sym, b, u, 8, 0.1, 128)
    c_rows = np.zeros(b.num_tokens, bool)
    for u, n in enumerate(lengths):
        r0 = int(b.tok_off_host[u])
        c_rows[r0:r0 + n - 8] = True
    np.testing.assert_allclose(sym["m"][c_rows], dense["m"][c_rows], rtol=1e-4, atol=1e-7)
    again = run_engine(b, 4, 8, 0.1, 128, engine=sym["engine"])
    assert np.array_equal(again["m"], sym["m"]) and np.array_equal(again["r"], sym["r"])
    assert np.array_equal(again["idx"], sym["idx"])


def test_symmetric_flag_rejections():
    with pytest.raises(RkvError) as ei:
        Engine(4, 8, 1, 1000, redundancy="closed", symmetric_gemm=True)
    assert ei.value.code == -2
    with pytest.raises(RkvError) as ei:
        Engine(4, 8, 1, 1000, redundancy="max", symmetric_gemm=True)
    assert ei.value.code == -2
    with pytest.raises(RkvError) as ei:
        Engine(4, 8, 1, 1000, single_cta_gemm=True, symmetric_gemm=True)
    assert ei.value.code == -2


@pytest.mark.parametrize("G,w,N", [(4, 8, 32768), (2, 8, 49152), (4, 8, 40000), (8, 8, 40000),
                                   (4, 8, 65536), (1, 8, 131072)])
def test_long_units(G, w, N):
    """Units longer than 32K tokens and up to 64 query rows; every tile of a
    unit's chunks streams through one pass (chunk exchanges in global memory)."""
    b = rand_batch([N], G, w, seed=1, dup=0.0)
    modes = ("closed", "gemm", "max", "gemm_sym") if N <= 65536 else ("closed", "gemm_sym")
    for mode in modes:
        out = run_engine(b, G, w, 0.1, 4096, mode=mode)
        check_unit(out, b, 0, w, 0.1, 4096, redundancy=oracle_mode(mode))
        del out


def test_rejects_too_long_unit_and_capacity():
    b = rand_batch([131073], 1, 8, seed=0, dup=0.0)
    eng = Engine(1, 8, max_units=1, max_tokens=b.num_tokens, redundancy="closed")
    a, r = eng.alloc_scores(b)
    with pytest.raises(RkvError) as ei:
        eng.score(b, a, r)
    assert ei.value.code == -2
    # a unit longer than the engine's declared max_unit_tokens
    b4 = rand_batch([5000], 4, 8, seed=0, dup=0.0)
    eng4 = Engine(4, 8, max_units=1, max_tokens=b4.num_tokens, redundancy="gemm",
                  symmetric_gemm=True, max_unit_tokens=4096)
    with pytest.raises(RkvError) as ei:
        eng4.score(b4, *eng4.alloc_scores(b4))
    assert ei.value.code == -2
    b2 = rand_batch([200], 1, 8, seed=0, dup=0.0)
    small = Engine(1, 8, max_units=1, max_tokens=100, redundancy="closed")
    with pytest.raises(RkvError) as ei:
        small.score(b2, a, r)
    assert ei.value.code == -6
    two = rand_batch([100, 100], 1, 8, seed=0, dup=0.0)
    with pytest.raises(RkvError) as ei:
        small.score(two, a, r)
    assert ei.value.code == -6
    bad = Batch(b.K, b.V, b.Q, np.array([0, 5]))   # N < w
    with pytest.raises(RkvError) as ei:
        eng.score(bad, a, r)
    assert ei.value.code == -1


def test_repeated_calls_are_deterministic():
    b = rand_batch([4000, 6000], 4, 8, seed=5)
    for mode in ("closed", "gemm", "max"):
        eng = Engine(4, 8, max_units=2, max_tokens=b.num_tokens, redundancy=mode)
        o1 = run_engine(b, 4, 8, 0.1, 512, engine=eng)
        o2 = run_engine(b, 4, 8, 0.1, 512, engine=eng)
        assert np.array_equal(o1["a"], o2["a"]) and np.array_equal(o1["r"], o2["r"])
        assert np.array_equal(o1["idx"], o2["idx"])


# ----------------------------------------------------------------- full workloads
def _sampled(name, n_sample, modes=("gemm", "closed")):
    wl = W.WORKLOADS[name]
    gb = W.generate(wl, seed=0, device=DEV)
    b = make_batch(gb)
    U = b.num_units
    rng = np.random.default_rng(123)
    units = sorted(set([0, U - 1] + rng.choice(U, size=min(U, n_sample), replace=False).tolist()))
    for mode in modes:
        for lam in wl.lambdas:
            out = run_engine(b, wl.group, wl.window, lam, wl.budget, mode=mode)
            for u in units:
                check_unit(out, b, u, wl.window, lam, wl.budget, redundancy=oracle_mode(mode))
            del out
            torch.cuda.empty_cache()
    return b, units


def test_workload_tiny_full():
    _sampled("tiny", 1, modes=("gemm", "closed", "max"))


def test_workload_llama3_layer_full():
    _sampled("llama3_8b_layer", 8, modes=("gemm", "closed", "max", "gemm_sym"))


def test_workload_r1_cadence_sampled():
    # the R1-Llama-8B cache at its trigger: B + 128 = 2176 tokens per unit
    _sampled("r1_llama8b_cadence", 6, modes=("gemm_sym", "closed"))


def test_workload_tiny_definition_redundancy():
    """Redundancy checked against the row-block definition (not the closed form)."""
    wl = W.WORKLOADS["tiny"]
    b = make_batch(W.generate(wl, seed=1, device=DEV))
    out = run_engine(b, wl.group, wl.window, 0.1, wl.budget, mode="gemm")
    check_unit(out, b, 0, wl.window, 0.1, wl.budget, redundancy="rowblocks")


@pytest.mark.slow
def test_workload_r1_llama8b_cache_sampled():
    _sampled("r1_llama8b_cache", 6, modes=("gemm", "closed", "gemm_sym"))


@pytest.mark.slow
def test_workload_long_trace_32k_sampled():
    _sampled("long_trace_32k", 6, modes=("gemm", "closed", "gemm_sym"))


@pytest.mark.slow
def test_workload_ragged_serving_sampled():
    _sampled("ragged_serving", 8, modes=("gemm", "closed", "max", "gemm_sym"))


@pytest.mark.slow
@pytest.mark.parametrize("name,mode", [("r1_llama8b_cache", "gemm_sym"),
                                       ("long_trace_32k", "gemm_sym"),
                                       ("long_trace_32k", "closed"),
                                       ("ragged_serving", "gemm_sym"),
                                       ("ragged_serving", "closed")])
def test_workload_all_units(name, mode):
    """Every unit of the full-size workload (the bench's inputs, seed 0) against
    the oracle, at each of the workload's lambdas (0, 0.1 and 1 for the ragged
    serving batch)."""
    wl = W.WORKLOADS[name]
    b = make_batch(W.generate(wl, seed=0, device=DEV))
    assert check_all_units(b, wl.group, wl.window, wl.budget, wl.lambdas, mode) == wl.num_units
