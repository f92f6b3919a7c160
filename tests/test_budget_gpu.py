"""Selection with attention sinks and per-unit budgets (rkv_select_ex) and the
ReFreeKV adaptive budget (rkv_refree_budget) on the GPU, against the oracle."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Engine, RkvError
from decode_kv_cache_eviction_b200 import workloads as W
from oracle import rkv_oracle as ora

from parity import close, make_batch, rand_batch, unit_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("sinks", [0, 4, 100])
@pytest.mark.parametrize("lam", [0.0, 0.1])
def test_select_ex_bit_exact_given_scores(sinks, lam):
    lengths = [8, 9, 50, 1000, 4096, 300, 20000, 130]
    w, budget = 8, 256
    b = rand_batch(lengths, 1, w, seed=sinks + 3)
    rng = np.random.default_rng(sinks)
    T = b.num_tokens
    a = (rng.random(T) * 1e-3).astype(np.float32)
    r = (rng.random(T) * 1e-3).astype(np.float32)
    a[::5] = a[2]
    r[::5] = r[2]
    U = len(lengths)
    budgets = rng.integers(0, budget + 1, U).astype(np.int32)
    budgets[0], budgets[1], budgets[2] = 0, budget, 3
    budgets[3] = 10**6                    # clamped to budget
    eng = Engine(1, w, max_units=U, max_tokens=T, redundancy="closed")
    ta, tr = torch.from_numpy(a).to(DEV), torch.from_numpy(r).to(DEV)
    Wd = budget + sinks + w
    idx = torch.full((U, Wd), 7, dtype=torch.int32, device=DEV)
    nk = torch.empty(U, dtype=torch.int32, device=DEV)
    eng.select_ex(b, ta, tr, lam, budget, idx, nk, torch.from_numpy(budgets).to(DEV), sinks)
    eng.check_status()
    idx, nk = idx.cpu().numpy(), nk.cpu().numpy()
    lam32 = np.float32(lam)
    for u, N in enumerate(lengths):
        r0 = int(b.tok_off_host[u])
        s32 = ora.joint_score(a[r0:r0 + N - w], r[r0:r0 + N - w], lam32)
        B = int(min(max(budgets[u], 0), budget))
        want = ora.select_with_sinks(s32, N, w, B, sinks)
        assert nk[u] == len(want), u
        np.testing.assert_array_equal(idx[u, :nk[u]], want)
        assert np.all(idx[u, nk[u]:] == -1)


def test_select_ex_without_extras_equals_select():
    lengths = [1000, 4096, 300, 9]
    b = rand_batch(lengths, 1, 8, seed=77)
    rng = np.random.default_rng(1)
    a = torch.from_numpy((rng.random(b.num_tokens) * 1e-3).astype(np.float32)).to(DEV)
    r = torch.from_numpy((rng.random(b.num_tokens) * 1e-3).astype(np.float32)).to(DEV)
    eng = Engine(1, 8, max_units=4, max_tokens=b.num_tokens, redundancy="closed")
    i1, n1, _, _ = eng.alloc_outputs(b, 200)
    i2, n2, _, _ = eng.alloc_outputs(b, 200)
    eng.select(b, a, r, 0.1, 200, i1, n1)
    eng.select_ex(b, a, r, 0.1, 200, i2, n2)
    torch.cuda.synchronize()
    assert torch.equal(i1, i2) and torch.equal(n1, n2)


def check_refree(b, G, w, T, sinks, max_budget, p_last, budgets, keep):
    p_last = p_last.cpu().numpy()
    budgets = budgets.cpu().numpy()
    keep = keep.cpu().numpy()
    for u in range(b.num_units):
        k_, _, q = unit_inputs(b, u)
        N = k_.shape[0]
        r0 = int(b.tok_off_host[u])
        p_o = ora.last_query_probs(q, k_)
        close(p_last[r0:r0 + N], p_o, f"unit {u} p_last")
        k_o = ora.refree_keep_count(p_o, sinks, T)
        kg = int(keep[u])
        if kg != k_o:
            # only a near tie at the stopping point may move it
            m = min(sinks, N)
            order = np.concatenate([np.arange(m), np.arange(N - 1, m - 1, -1)])
            cum = np.cumsum(p_o[order] ** 2)
            need = (1 - T) ** 2 * cum[-1]
            lo, hi = min(kg, k_o), max(kg, k_o)
            assert abs(cum[lo - 1] - need) <= 2e-4 * need or abs(cum[hi - 1] - need) <= 2e-4 * need, \
                (u, kg, k_o)
        assert int(budgets[u]) == min(ora.refree_budget(kg, N, w, sinks), max_budget)


@pytest.mark.parametrize("G,w", [(1, 8), (2, 4), (4, 8), (5, 3), (8, 2)])
@pytest.mark.parametrize("T", [0.01, 0.2])
def test_refree_budget_matches_oracle(G, w, T):
    lengths = [w, w + 1, 100, 1000, 5000, 2500]
    b = rand_batch(lengths, G, w, seed=G * 7 + w)
    # scale queries so that attention is peaked, as in a trained model
    b.Q.mul_(3.0)
    eng = Engine(G, w, max_units=len(lengths), max_tokens=b.num_tokens, redundancy="closed")
    p_last = torch.full((b.num_tokens,), float("nan"), device=DEV)
    budgets = torch.empty(len(lengths), dtype=torch.int32, device=DEV)
    keep = torch.empty(len(lengths), dtype=torch.int32, device=DEV)
    eng.refree_budget(b, T, 4, 4096, p_last, budgets, keep)
    eng.check_status()
    check_refree(b, G, w, T, 4, 4096, p_last, budgets, keep)


def test_refree_rejects_large_groups():
    b = rand_batch([100], 16, 2, seed=1)
    eng = Engine(16, 2, max_units=1, max_tokens=100, redundancy="closed")
    p = torch.empty(100, device=DEV)
    bud = torch.empty(1, dtype=torch.int32, device=DEV)
    with pytest.raises(RkvError) as ei:
        eng.refree_budget(b, 0.01, 4, 64, p, bud)
    assert ei.value.code == -2


def test_adaptive_budget_pipeline_llama3_layer():
    """refree budget -> selection with sinks and per-unit budgets -> compaction,
    kept sets against the oracle (near ties excepted)."""
    wl = W.WORKLOADS["llama3_8b_layer"]
    b = make_batch(W.generate(wl, seed=2, device=DEV))
    G, w, sinks, T, maxb = wl.group, wl.window, 4, 0.01, 2048
    eng = Engine(G, w, max_units=b.num_units, max_tokens=b.num_tokens, redundancy="gemm")
    p_last = torch.empty(b.num_tokens, device=DEV)
    budgets = torch.empty(b.num_units, dtype=torch.int32, device=DEV)
    keep = torch.empty(b.num_units, dtype=torch.int32, device=DEV)
    eng.refree_budget(b, T, sinks, maxb, p_last, budgets, keep)
    a, r = eng.alloc_scores(b)
    eng.score(b, a, r)
    Wd = maxb + sinks + w
    idx = torch.empty((b.num_units, Wd), dtype=torch.int32, device=DEV)
    nk = torch.empty(b.num_units, dtype=torch.int32, device=DEV)
    eng.select_ex(b, a, r, 0.1, maxb, idx, nk, budgets, sinks)
    Ko, Vo = (torch.empty((b.num_units, Wd, 128), dtype=torch.bfloat16, device=DEV)
              for _ in range(2))
    eng.compact(b, idx, nk, maxb + sinks, Ko, Vo)
    eng.check_status()
    torch.cuda.synchronize()
    check_refree(b, G, w, T, sinks, maxb, p_last, budgets, keep)
    bud = budgets.cpu().numpy()
    idx, nk = idx.cpu().numpy(), nk.cpu().numpy()
    for u in range(b.num_units):
        k_, _, q = unit_inputs(b, u)
        N = k_.shape[0]
        _, a_o = ora.importance(q, k_)
        _, r_o = ora.redundancy_mean(k_, w)
        s_o = ora.joint_score(a_o, r_o, 0.1)
        want = ora.select_with_sinks(s_o, N, w, int(bud[u]), sinks)
        got = idx[u, :nk[u]]
        assert len(got) == len(want)
        diff = set(got.tolist()) ^ set(want.tolist())
        if diff:
            assert int(bud[u]) >= 1, u
            m = min(sinks, N - w)
            sb = np.sort(s_o[m:])[::-1][int(bud[u]) - 1]
            band = 1e-5 * np.max(np.abs(s_o))
            assert all(abs(s_o[i] - sb) <= band for i in diff), u
        r0 = int(b.tok_off_host[u])
        src = torch.from_numpy(got.astype(np.int64) + r0).to(DEV)
        assert torch.equal(Ko[u, :nk[u]].view(torch.int16), b.K[src].view(torch.int16))
