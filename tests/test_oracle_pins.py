"""Pins for the fp64 oracle: things other than the oracle itself that fix what
it must compute (R-KV article, "R-KV三步走": 重要性打分, 冗余打分, 联合淘汰).

* a hand-derived 6-token worked example (tests/golden/worked_6token.json);
* a second, loop-only transcription on tiny inputs;
* textbook special cases (w = 1, G = 1 reduces importance to a plain softmax,
  checked against scipy);
* brute force over every budget-subset for N <= 12;
* invariants: B >= N - w keeps everything, lambda = 1 is pure attention top-B,
  lambda = 0 keeps the least redundant, permutation equivariance, cosine scale
  invariance, exact duplicates tie, heavily repeated keys are the most
  redundant, GQA averaging is linear in the heads;
* mutation checks: a planted mistake in a copy of the oracle fails the pins.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import loops
from oracle import rkv_oracle as ora

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_6token.json")


def _worked():
    with open(GOLD) as f:
        g = json.load(f)
    K = np.array(g["K"], dtype=np.float64)
    Q = np.array(g["Q"], dtype=np.float64).reshape(g["group"], g["window"], g["d"])
    return g, Q, K


def check_worked_example(o):
    """Return a list of mismatches of oracle module ``o`` against the fixture."""
    g, Q, K = _worked()
    w, B, tol = g["window"], g["budget"], g["tolerance"]
    bad = []
    p = o.attention_probs(Q, K)[0]
    if not np.allclose(p, g["p"], atol=tol, rtol=0):
        bad.append("p")
    abar, a = o.importance(Q, K)
    if not np.allclose(abar, g["abar"], atol=tol, rtol=0):
        bad.append("abar")
    if not np.allclose(a, g["a"], atol=tol, rtol=0):
        bad.append("a")
    for fn in (o.redundancy_mean, o.redundancy_mean_closed_form):
        m, r = fn(K, w)
        if not np.allclose(m, g["m"], atol=tol, rtol=0):
            bad.append(fn.__name__ + ".m")
        if not np.allclose(r, g["r"], atol=tol, rtol=0):
            bad.append(fn.__name__ + ".r")
    m, r = o.redundancy_mean(K, w)
    s = o.joint_score(a, r, 0.1)
    if not np.allclose(s, g["s"]["0.1"], atol=tol, rtol=0):
        bad.append("s")
    for lam, want in g["idx"].items():
        s = o.joint_score(a, r, float(lam))
        idx = o.select(s, K.shape[0], w, B)
        if list(idx) != want:
            bad.append("idx@" + lam)
    return bad


def test_worked_example():
    assert check_worked_example(ora) == []


def test_worked_example_through_run_unit():
    g, Q, K = _worked()
    V = np.arange(12, dtype=np.float64).reshape(6, 2)
    out = ora.run_unit(Q, K, V, g["window"], g["budget"], 0.1)
    assert list(out["idx"]) == g["idx"]["0.1"]
    np.testing.assert_array_equal(out["V"], V[[2, 3, 4, 5]])
    np.testing.assert_array_equal(out["K"], K[[2, 3, 4, 5]])


def _rand_unit(rng, N, d, G, w, dup=0.0):
    K = rng.standard_normal((N, d))
    if dup:
        for i in range(1, N):
            if rng.random() < dup:
                K[i] = K[rng.integers(0, i)]
    Q = rng.standard_normal((G, w, d))
    return Q, K


@pytest.mark.parametrize("seed", range(12))
def test_matches_loop_transcription(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(4, 40))
    w = int(rng.integers(1, min(N - 1, 6) + 1))
    d = int(rng.choice([2, 3, 8, 16]))
    G = int(rng.integers(1, 4))
    B = int(rng.integers(0, N))
    lam = float(rng.choice([0.0, 0.1, 0.5, 1.0]))
    Q, K = _rand_unit(rng, N, d, G, w, dup=0.2)
    V = rng.standard_normal((N, d))
    ref = loops.run_unit(Q.tolist(), K.tolist(), w, B, lam)
    out = ora.run_unit(Q, K, V, w, B, lam)
    np.testing.assert_allclose(out["abar"], ref["abar"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["a"], ref["a"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["m"], ref["m"], rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(out["r"], ref["r"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out["s"], ref["s"], rtol=1e-10, atol=1e-14)
    assert list(out["idx"]) == ref["idx"]


@pytest.mark.parametrize("N", [300, 2049, 4100])
def test_closed_form_equals_definition(N):
    rng = np.random.default_rng(N)
    K = rng.standard_normal((N, 128)) * rng.uniform(0.5, 4, size=128)
    K[5] = K[3]          # an exact duplicate
    K[7] = 0.0           # a zero key
    m1, r1 = ora.redundancy_mean(K, 8, block=512)
    m2, r2 = ora.redundancy_mean_closed_form(K, 8)
    np.testing.assert_allclose(m2, m1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r2, r1, rtol=1e-10, atol=0)
    assert m1[7] == 0.0


@pytest.mark.parametrize("N", [1, 17, 512])
def test_single_query_is_textbook_softmax(N):
    rng = np.random.default_rng(N)
    d = 128
    K = rng.standard_normal((N, d))
    Q = rng.standard_normal((1, 1, d))
    abar, a = ora.importance(Q, K)
    want = scipy.special.softmax(K @ Q[0, 0] / math.sqrt(d))
    np.testing.assert_allclose(abar, want, rtol=1e-12)
    if N > 1:
        np.testing.assert_allclose(a, want[:-1] / want[:-1].sum(), rtol=1e-12)


def test_causal_mask_hides_later_keys():
    rng = np.random.default_rng(3)
    Q, K = _rand_unit(rng, 20, 8, 2, 4)
    p = ora.attention_probs(Q, K)
    for t in range(4):
        last = 20 - 4 + t
        assert np.all(p[:, t, last + 1:] == 0)
        assert np.all(p[:, t, :last + 1] > 0)
        np.testing.assert_allclose(p[:, t].sum(axis=1), 1.0, rtol=1e-13)


def test_gqa_average_is_linear_in_heads():
    rng = np.random.default_rng(4)
    Q, K = _rand_unit(rng, 50, 16, 3, 4)
    abar, _ = ora.importance(Q, K)
    per_head = [ora.importance(Q[g:g + 1], K)[0] for g in range(3)]
    np.testing.assert_allclose(abar, np.mean(per_head, axis=0), rtol=1e-13)


@pytest.mark.parametrize("seed", range(6))
def test_selection_matches_subset_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(5, 13))
    w = int(rng.integers(1, 4))
    B = int(rng.integers(1, N - w + 1))
    Q, K = _rand_unit(rng, N, 4, 2, w, dup=0.3)
    for lam in (0.0, 0.1, 1.0):
        _, a = ora.importance(Q, K)
        _, r = ora.redundancy_mean(K, w)
        s = ora.joint_score(a, r, lam)
        assert list(ora.select(s, N, w, B)) == loops.select_by_subsets(
            s.tolist(), N, w, B)


def test_ties_break_to_lower_index():
    s = np.array([0.5, 0.2, 0.5, 0.5, 0.1])
    assert list(ora.select(s, 7, 2, 2)) == [0, 2, 5, 6]
    assert list(ora.select(s, 7, 2, 3)) == [0, 2, 3, 5, 6]


@pytest.mark.parametrize("B", [6, 7, 100])
def test_budget_at_least_candidates_keeps_all(B):
    rng = np.random.default_rng(B)
    Q, K = _rand_unit(rng, 12, 8, 1, 6)
    out = ora.run_unit(Q, K, K, 6, B, 0.1)
    assert list(out["idx"]) == list(range(12))


def test_lambda_one_is_pure_attention_topB():
    rng = np.random.default_rng(7)
    Q, K = _rand_unit(rng, 400, 32, 4, 8)
    out = ora.run_unit(Q, K, K, 8, 50, 1.0)
    _, a = ora.importance(Q, K)
    thr = np.sort(a)[::-1][49]
    kept = out["idx"][:-8]
    assert len(kept) == 50 and np.all(a[kept] >= thr)
    assert np.all(np.delete(a, kept) <= thr)


def test_lambda_zero_keeps_least_redundant():
    rng = np.random.default_rng(8)
    Q, K = _rand_unit(rng, 400, 32, 4, 8, dup=0.2)
    out = ora.run_unit(Q, K, K, 8, 60, 0.0)
    m, _ = ora.redundancy_mean_closed_form(K, 8)
    kept = out["idx"][:-8]
    assert m[kept].max() <= np.delete(m, kept).min() + 1e-15


def test_candidate_permutation_equivariance():
    rng = np.random.default_rng(9)
    N, w, B = 300, 8, 40
    Q, K = _rand_unit(rng, N, 16, 2, w)
    V = rng.standard_normal((N, 16))
    perm = np.concatenate([rng.permutation(N - w), np.arange(N - w, N)])
    o1 = ora.run_unit(Q, K, V, w, B, 0.1)
    o2 = ora.run_unit(Q, K[perm], V[perm], w, B, 0.1)
    np.testing.assert_allclose(o2["a"], o1["a"][perm[:N - w]], rtol=1e-12)
    np.testing.assert_allclose(o2["r"], o1["r"][perm[:N - w]], rtol=1e-12)
    # kept sets map onto each other (no exact ties in continuous random data)
    kept1 = set(o1["idx"][:-w].tolist())
    kept2 = set(perm[o2["idx"][:-w]].tolist())
    assert kept1 == kept2


def test_cosine_scale_invariance():
    rng = np.random.default_rng(10)
    K = rng.standard_normal((200, 32))
    m1, r1 = ora.redundancy_mean(K, 4)
    m2, r2 = ora.redundancy_mean(K * rng.uniform(0.1, 10, size=(200, 1)), 4)
    np.testing.assert_allclose(m2, m1, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(r2, r1, rtol=1e-11)


def test_exact_duplicates_tie_and_repeats_are_most_redundant():
    rng = np.random.default_rng(11)
    # margin of a 16-fold key: 15/(N-1) ~ 0.05; spread of m among i.i.d.
    # keys: 1/sqrt(d N) ~ 0.005, so the repeats must top the ranking
    N, d = 300, 128
    K = rng.standard_normal((N, d))
    rep = list(range(10, 290, 18))                       # 16 copies of key 10
    K[rep] = K[10]
    K[20] = 3.0 * K[30]                                  # same direction
    m, r = ora.redundancy_mean(K, 8)
    # identical up to the summation order of the BLAS row blocks
    np.testing.assert_allclose(m[rep], m[rep[0]], rtol=1e-13, atol=0)
    np.testing.assert_allclose(r[rep], r[rep[0]], rtol=1e-13, atol=0)
    assert m[20] == pytest.approx(m[30], abs=1e-15)
    assert set(np.argsort(m)[::-1][:len(rep)].tolist()) == set(rep)


def test_degenerate_no_candidates():
    rng = np.random.default_rng(12)
    Q, K = _rand_unit(rng, 6, 4, 1, 6)
    out = ora.run_unit(Q, K, K, 6, 3, 0.1)
    assert out["a"].size == 0 and out["r"].size == 0
    assert list(out["idx"]) == list(range(6))


# ---- mutation checks: each planted mistake must fail a pin ----------------

class _Mutant:
    def __init__(self, **over):
        for k in dir(ora):
            if not k.startswith("__"):
                setattr(self, k, getattr(ora, k))
        for k, v in over.items():
            setattr(self, k, v)


def _no_causal_mask(Q, K):
    G, w, d = Q.shape
    z = np.einsum("gtd,nd->gtn", Q, K) / np.sqrt(d)
    e = np.exp(z - z.max(axis=2, keepdims=True))
    return e / e.sum(axis=2, keepdims=True)


def _no_scale(Q, K):
    return ora.attention_probs(Q * np.sqrt(Q.shape[2]), K)


def _diag_kept(K, w, block=2048):
    N = K.shape[0]
    kh = ora.unit_keys(K)
    m = (kh[:N - w] @ kh.T).sum(axis=1) / (N - 1)
    return m, ora.softmax(m)


def _not_normalised(K, w, block=2048):
    N = K.shape[0]
    S = K[:N - w] @ K.T
    S[np.arange(N - w), np.arange(N - w)] = 0
    m = S.sum(axis=1) / (N - 1)
    return m, ora.softmax(m)


def _wrong_sign(a, r, lam):
    return lam * a + (1 - lam) * r


def _ties_high(s, N, w, budget):
    c = N - w
    if c <= budget:
        return np.arange(N)
    order = np.lexsort((-np.arange(c), -s))
    return np.concatenate([np.sort(order[:budget]), np.arange(c, N)])


@pytest.mark.parametrize("over", [
    dict(attention_probs=_no_causal_mask),
    dict(attention_probs=_no_scale),
    dict(redundancy_mean=_diag_kept, redundancy_mean_closed_form=_diag_kept),
    dict(redundancy_mean=_not_normalised,
         redundancy_mean_closed_form=_not_normalised),
    dict(joint_score=_wrong_sign),
    dict(select=_ties_high),
], ids=["no-causal-mask", "no-1/sqrt(d)", "diagonal-kept", "raw-dot-not-cosine",
        "wrong-sign", "ties-to-high-index"])
def test_planted_mistake_fails_worked_example(over):
    assert check_worked_example(_Mutant(**over)) != []


# ---- row-max redundancy (nearest duplicate) --------------------------------

@pytest.mark.parametrize("seed", range(6))
def test_row_max_matches_loop_transcription(seed):
    rng = np.random.default_rng(200 + seed)
    N = int(rng.integers(3, 40))
    w = int(rng.integers(1, min(N - 1, 5) + 1))
    Q, K = _rand_unit(rng, N, 8, 1, w, dup=0.2)
    m_ref, r_ref = loops.redundancy_max(K.tolist(), w)
    m, r = ora.redundancy_max(K, w, block=7)
    np.testing.assert_allclose(m, m_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r, r_ref, rtol=1e-12)


def test_row_max_exact_duplicates_are_maximal():
    rng = np.random.default_rng(21)
    K = rng.standard_normal((500, 128))
    K[100] = K[7]
    K[300] = 2.5 * K[40]          # same direction counts as a duplicate
    m, r = ora.redundancy_max(K, 8)
    assert m[7] == pytest.approx(1.0, abs=1e-12) and m[100] == pytest.approx(1.0, abs=1e-12)
    assert m[40] == pytest.approx(1.0, abs=1e-12) and m[300] == pytest.approx(1.0, abs=1e-12)
    others = np.delete(m, [7, 100, 40, 300])
    assert others.max() < 0.6      # i.i.d. 128-d keys are far from each other
    assert r[7] == pytest.approx(r.max(), rel=1e-12)


def test_row_max_worked_example():
    g, Q, K = _worked()
    # unit keys (1,0),(1,0),(0,1),(-1,0),(1,1)/sqrt2,(0,-1): nearest other key of
    # each candidate, by hand: k0 ~ k1 (1), k1 ~ k0 (1), k2 ~ k4 (1/sqrt2), k3 ~ k2 (0)
    m, _ = ora.redundancy_max(K, g["window"])
    np.testing.assert_allclose(m, [1.0, 1.0, 1 / np.sqrt(2), 0.0], atol=1e-12)


def test_row_max_zero_key_and_window_keys_count():
    K = np.array([[1.0, 0.0], [0.0, 0.0], [0.0, 1.0], [1.0, 0.0]])
    m, _ = ora.redundancy_max(K, 1)   # candidates 0..2; key 3 (window) duplicates key 0
    np.testing.assert_allclose(m, [1.0, 0.0, 0.0], atol=1e-15)


# ---- in-place slot reuse (eviction mask + free slots) -----------------------

@pytest.mark.parametrize("seed", range(5))
def test_evict_in_place_matches_scan_and_partitions_slots(seed):
    rng = np.random.default_rng(300 + seed)
    N = int(rng.integers(2, 300))
    w = int(rng.integers(1, min(N, 8) + 1))
    s = rng.standard_normal(N - w)
    budget = int(rng.integers(0, N))
    idx = ora.select(s, N, w, budget)
    keep, free = ora.evict_in_place(N, idx)
    keep_l, free_l = loops.evict_in_place(N, idx.tolist())
    assert keep.tolist() == keep_l and free.tolist() == free_l
    # kept and free slots partition 0..N-1; free is ascending; the window is live
    assert sorted(idx.tolist() + free.tolist()) == list(range(N))
    assert np.all(np.diff(free) > 0)
    assert keep[N - w:].all()
    assert keep.sum() == len(idx)


def test_in_place_live_rows_equal_gather_compaction():
    """Reading the live slots in ascending order gives exactly the rows that
    gather compaction writes."""
    rng = np.random.default_rng(31)
    Q, K = _rand_unit(rng, 400, 16, 2, 4, dup=0.2)
    V = rng.standard_normal(K.shape)
    out = ora.run_unit(Q, K, V, 4, 50, 0.1, redundancy="closed")
    keep, free = ora.evict_in_place(400, out["idx"])
    np.testing.assert_array_equal(K[keep], out["K"])
    np.testing.assert_array_equal(V[keep], out["V"])
    assert len(free) == 400 - len(out["idx"])


def test_fill_free_slots_takes_lowest_slots_first():
    K = np.arange(10 * 3, dtype=np.float64).reshape(10, 3)
    V = -K
    keep, free = ora.evict_in_place(10, np.array([1, 4, 5, 8, 9]))
    assert free.tolist() == [0, 2, 3, 6, 7]
    Kn = np.full((3, 3), 100.0) + np.arange(3)[:, None]
    K2, V2, keep2 = ora.fill_free_slots(K, V, keep, free, Kn, -Kn)
    assert np.array_equal(K2[[0, 2, 3]], Kn) and np.array_equal(V2[[0, 2, 3]], -Kn)
    untouched = [1, 4, 5, 6, 7, 8, 9]
    assert np.array_equal(K2[untouched], K[untouched])
    assert keep2.tolist() == [True, True, True, True, True, True, False, False, True, True]
    with pytest.raises(AssertionError):
        ora.fill_free_slots(K, V, keep, free, np.zeros((6, 3)), np.zeros((6, 3)))


# ---- sinks + per-unit budgets; ReFreeKV adaptive budget ----------------------

@pytest.mark.parametrize("seed", range(6))
def test_select_with_sinks_reduces_and_brute_force(seed):
    rng = np.random.default_rng(400 + seed)
    N = int(rng.integers(3, 13))
    w = int(rng.integers(1, 3))
    s = np.round(rng.standard_normal(N - w), 1)       # ties on purpose
    for budget in range(0, N - w + 1):
        assert np.array_equal(ora.select_with_sinks(s, N, w, budget, 0),
                              ora.select(s, N, w, budget))
        for sinks in (1, 2, 4):
            got = ora.select_with_sinks(s, N, w, budget, sinks).tolist()
            m = min(sinks, N - w)
            # sinks and window always kept; the middle is the brute-force best subset
            assert got[:m] == list(range(m)) and got[-w:] == list(range(N - w, N))
            mid = got[m:len(got) - w]
            if N - w - m <= budget:
                assert got == list(range(N))
            else:
                sub = loops.select_by_subsets(list(s[m:]), N - m, w, budget)
                assert mid == [i + m for i in sub[:budget]]


def test_last_query_probs_is_last_row_of_attention():
    rng = np.random.default_rng(9)
    Q, K = _rand_unit(rng, 50, 8, 3, 4)
    p = ora.last_query_probs(Q, K)
    assert p.shape == (50,) and abs(p.sum() - 1.0) < 1e-12
    # the newest query sees every key: with w = 1, G = 1 it is a plain softmax
    from scipy.special import softmax as sp_softmax
    Q1 = Q[:1, -1:, :]
    np.testing.assert_allclose(ora.last_query_probs(Q1, K),
                               sp_softmax(K @ Q1[0, 0] / np.sqrt(8)), rtol=1e-12)


def test_refree_keep_count_closed_forms():
    N = 1000
    # uniform row: norm of the first k entries is sqrt(k/N) of the full norm
    p = np.full(N, 1.0 / N)
    for T in (0.01, 0.013, 0.37):     # (1 - T)^2 N away from an integer
        want = int(np.ceil((1 - T) ** 2 * N))
        assert ora.refree_keep_count(p, 4, T) == want
    # all mass on the sinks: the sinks alone suffice
    p = np.zeros(N); p[:4] = 0.25
    assert ora.refree_keep_count(p, 4, 0.01) == 4
    # all mass on the newest token: sinks (ranked first) plus that one
    p = np.zeros(N); p[-1] = 1.0
    assert ora.refree_keep_count(p, 4, 0.01) == 5
    assert ora.refree_keep_count(p, 0, 0.01) == 1
    # one old token holds all the mass: everything back to it is kept
    p = np.zeros(N); p[100] = 1.0
    assert ora.refree_keep_count(p, 4, 0.01) == 4 + (N - 100)


def _keep_cut_norm(p, sinks, T):
    """A rejected reading: stop once the cut-off entries' norm is at most T of
    the row's norm (planted here only to show that the pins tell it apart)."""
    N = len(p)
    m = min(sinks, N)
    order = np.concatenate([np.arange(m), np.arange(N - 1, m - 1, -1)])
    e = p[order] ** 2
    cut = e.sum() - np.cumsum(e)
    return int(np.argmax(np.sqrt(np.maximum(cut, 0)) <= T * np.sqrt(e.sum()))) + 1


def _keep_cut_energy(p, sinks, T):
    """Another rejected reading: the cut-off entries' squared norm at most T of
    the row's squared norm."""
    N = len(p)
    m = min(sinks, N)
    order = np.concatenate([np.arange(m), np.arange(N - 1, m - 1, -1)])
    e = p[order] ** 2
    cut = e.sum() - np.cumsum(e)
    return int(np.argmax(cut <= T * e.sum())) + 1


def test_refree_reading_is_the_drop_of_the_frobenius_norm():
    """ReFreeKV review, section 2 ("Uni-Metric"): the metric is the Frobenius
    norm of the kept attention entries, which the review calls their energy;
    cutting stops once the energy lost, the drop of that norm, is under T.
    Hand-worked values, with the two rejected readings giving other counts."""
    # uniform 1000-token row, T = 1%: the kept norm is sqrt(k / 1000) of the
    # row's, and sqrt(k / 1000) >= 0.99 first holds at k = 981 (980.1 rounded up)
    p = np.full(1000, 1e-3)
    assert ora.refree_keep_count(p, 0, 0.01) == 981
    assert loops.refree_keep_count(list(p), 0, 0.01) == 981
    assert _keep_cut_norm(p, 0, 0.01) == 1000     # sqrt((1000 - k) / 1000) <= 0.01
    assert _keep_cut_energy(p, 0, 0.01) == 990    # (1000 - k) / 1000 <= 0.01
    # five tokens, one sink, T = 0.1.  Ranking: 0 (sink), 4, 3, 2, 1.
    # Squares: 0.01, 0.04, 0.09, 0.0225, 0.0625, total 0.225; the kept prefix
    # needs 0.81 * 0.225 = 0.18225: {0} 0.01, {0,4} 0.0725, {0,4,3} 0.095,
    # {0,4,3,2} 0.185 -> 4 tokens.  Cutting token 1 alone removes 0.04 of
    # squared norm, more than 0.01 * 0.225 and 0.1 * 0.225, so both rejected
    # readings keep all 5.
    p5 = np.array([0.1, 0.2, 0.3, 0.15, 0.25])
    assert ora.refree_keep_count(p5, 1, 0.1) == 4
    assert loops.refree_keep_count(list(p5), 1, 0.1) == 4
    assert _keep_cut_norm(p5, 1, 0.1) == 5
    assert _keep_cut_energy(p5, 1, 0.1) == 5
    # the budget that keeps those 4 tokens of a unit with w = 1: 4 - 1 sink - 1
    assert ora.refree_budget(4, 5, 1, 1) == 2


@pytest.mark.parametrize("seed", range(4))
def test_refree_keep_count_matches_loop(seed):
    rng = np.random.default_rng(500 + seed)
    N = int(rng.integers(5, 400))
    p = rng.random(N) ** 8
    p /= p.sum()
    for T in (0.01, 0.05, 0.3):
        for sinks in (0, 4):
            assert ora.refree_keep_count(p, sinks, T) == loops.refree_keep_count(list(p), sinks, T)


def test_refree_budget_counts_sinks_and_window():
    assert ora.refree_budget(100, 1000, 8, 4) == 88
    assert ora.refree_budget(10, 1000, 8, 4) == 0
    assert ora.refree_budget(5, 6, 8 - 6 + 4, 4) == 0
