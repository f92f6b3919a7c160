"""In-place slot reuse on the GPU (rkv_evict_in_place, rkv_fill_slots) against
the oracle's evict_in_place / fill_free_slots, bit for bit, on the engine's own
kept indices."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Engine, RkvError
from decode_kv_cache_eviction_b200 import workloads as W
from oracle import rkv_oracle as ora

from parity import make_batch, rand_batch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def select_and_evict(b, G, w, budget, lam=0.1, mode="closed"):
    eng = Engine(G, w, max_units=b.num_units, max_tokens=b.num_tokens, redundancy=mode)
    a, r = eng.alloc_scores(b)
    idx, nk, Ko, Vo = eng.alloc_outputs(b, budget)
    eng.score(b, a, r)
    eng.select(b, a, r, lam, budget, idx, nk)
    eng.compact(b, idx, nk, budget, Ko, Vo)
    keep, free, nfree = eng.alloc_in_place(b)
    keep.fill_(9)
    free.fill_(-7)
    eng.evict_in_place(b, idx, nk, budget, keep, free, nfree)
    eng.check_status()
    torch.cuda.synchronize()
    return eng, dict(idx=idx.cpu().numpy(), nk=nk.cpu().numpy(), Ko=Ko, Vo=Vo, keep=keep,
                     free=free, nfree=nfree)


def check_evict(b, out):
    keep = out["keep"].cpu().numpy()
    free = out["free"].cpu().numpy()
    nfree = out["nfree"].cpu().numpy()
    for u in range(b.num_units):
        r0, r1 = int(b.tok_off_host[u]), int(b.tok_off_host[u + 1])
        N = r1 - r0
        kept = out["idx"][u, :out["nk"][u]]
        k_o, f_o = ora.evict_in_place(N, kept)
        assert np.array_equal(keep[r0:r1].astype(bool), k_o), u
        assert int(nfree[u]) == len(f_o)
        assert np.array_equal(free[r0:r0 + len(f_o)], f_o), u
        assert np.all(free[r0 + len(f_o):r1] == -1)
        # the live rows, read in slot order, are exactly what compaction gathers
        live = torch.from_numpy(np.flatnonzero(k_o) + r0).to(b.K.device)
        nk = int(out["nk"][u])
        assert torch.equal(b.K[live].view(torch.int16), out["Ko"][u, :nk].view(torch.int16))
        assert torch.equal(b.V[live].view(torch.int16), out["Vo"][u, :nk].view(torch.int16))


@pytest.mark.parametrize("budget", [0, 1, 64, 5000])
def test_evict_in_place_matches_oracle(budget):
    lengths = [8, 9, 127, 128, 129, 1000, 2500, 5000, 4104]
    b = rand_batch(lengths, 4, 8, seed=51 + budget)
    _, out = select_and_evict(b, 4, 8, budget)
    check_evict(b, out)


def test_evict_in_place_llama3_layer_workload():
    wl = W.WORKLOADS["llama3_8b_layer"]
    b = make_batch(W.generate(wl, seed=0, device=DEV))
    _, out = select_and_evict(b, wl.group, wl.window, wl.budget, mode="gemm")
    check_evict(b, out)


def test_evict_in_place_flags_bad_index():
    b = rand_batch([300, 200], 1, 4, seed=3)
    eng = Engine(1, 4, max_units=2, max_tokens=b.num_tokens, redundancy="closed")
    budget, Wd = 10, 14
    idx = np.full((2, Wd), -1, np.int32)
    idx[0, :3] = [5, 400, 7]          # 400 is outside unit 0 (N = 300)
    idx[1, :2] = [0, 199]
    nk = np.array([3, 2], np.int32)
    keep, free, nfree = eng.alloc_in_place(b)
    eng.evict_in_place(b, torch.from_numpy(idx).to(DEV), torch.from_numpy(nk).to(DEV), budget,
                       keep, free, nfree)
    with pytest.raises(RkvError) as ei:
        eng.check_status()
    assert ei.value.code == -7
    keep = keep.cpu().numpy()
    assert np.flatnonzero(keep[:300]).tolist() == [5, 7]      # the bad index is ignored
    assert np.flatnonzero(keep[300:]).tolist() == [0, 199]
    assert nfree.cpu().tolist() == [298, 198]


def test_fill_slots_matches_oracle_twice():
    lengths = [700, 300, 129, 2000]
    G, w, budget = 2, 8, 100
    b = rand_batch(lengths, G, w, seed=61)
    eng, out = select_and_evict(b, G, w, budget)
    rng = np.random.default_rng(5)
    # host-side expected state, unit by unit
    K = b.K.float().cpu().numpy()
    V = b.V.float().cpu().numpy()
    keep = out["keep"].cpu().numpy().astype(bool)
    frees = []
    for u in range(len(lengths)):
        r0, r1 = int(b.tok_off_host[u]), int(b.tok_off_host[u + 1])
        frees.append(ora.evict_in_place(r1 - r0, out["idx"][u, :out["nk"][u]])[1])
    for step in range(2):
        # at most the unit's free slots (overflow is its own test below)
        n_new = [int(rng.integers(0, len(frees[u]) + 1)) for u in range(len(lengths))]
        n_new[1] = min(5 + 10 * step, len(frees[1]))
        off = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int64)
        Kn = torch.randn(int(off[-1]), 128, device=DEV).to(torch.bfloat16)
        Vn = torch.randn(int(off[-1]), 128, device=DEV).to(torch.bfloat16)
        eng.fill_slots(b, off, Kn, Vn, out["keep"], out["free"], out["nfree"])
        eng.check_status()
        torch.cuda.synchronize()
        Knp, Vnp = Kn.float().cpu().numpy(), Vn.float().cpu().numpy()
        for u in range(len(lengths)):
            r0, r1 = int(b.tok_off_host[u]), int(b.tok_off_host[u + 1])
            sl = slice(int(off[u]), int(off[u + 1]))
            K2, V2, k2 = ora.fill_free_slots(K[r0:r1], V[r0:r1], keep[r0:r1], frees[u],
                                             Knp[sl], Vnp[sl])
            K[r0:r1], V[r0:r1], keep[r0:r1] = K2, V2, k2
            frees[u] = frees[u][n_new[u]:]
        assert np.array_equal(b.K.float().cpu().numpy(), K)
        assert np.array_equal(b.V.float().cpu().numpy(), V)
        assert np.array_equal(out["keep"].cpu().numpy().astype(bool), keep)
        fr = out["free"].cpu().numpy()
        for u in range(len(lengths)):
            r0 = int(b.tok_off_host[u])
            N = int(b.tok_off_host[u + 1]) - r0
            assert int(out["nfree"][u]) == len(frees[u])
            assert np.array_equal(fr[r0:r0 + len(frees[u])], frees[u])
            assert np.all(fr[r0 + len(frees[u]):r0 + N] == -1)


def test_fill_slots_more_tokens_than_free_slots():
    b = rand_batch([100, 50], 1, 8, seed=71)
    eng, out = select_and_evict(b, 1, 8, 80)     # unit 0: 12 free slots; unit 1: none
    assert out["nfree"].cpu().tolist() == [12, 0]
    off = np.array([0, 20, 23], np.int64)
    Kn = torch.randn(23, 128, device=DEV).to(torch.bfloat16)
    eng.fill_slots(b, off, Kn, Kn, out["keep"], out["free"], out["nfree"])
    with pytest.raises(RkvError) as ei:
        eng.check_status()
    assert ei.value.code == -7
    assert out["nfree"].cpu().tolist() == [0, 0]
    assert bool(out["keep"][:100].all())
