"""rkv_score_noalloc: scoring for callers that cannot allocate device memory.

Some callers own every byte of HBM through their own allocator (a serving stack
that reserves nearly all memory for its KV block pool up front) or load this
library as a plug-in that must not call cudaMalloc behind the host framework's
back; they cannot create an engine, whose workspace is allocated.  This call
gives them the GEMM-mode scores with the library's fixed static device scratch
instead.  Its results must agree with the engine path and with the fp64 oracle
(the tolerance of every parity test: 1e-6 absolute + 1e-3 relative) on
consecutive calls, since every call reuses the same static scratch, and a
call must not change the device's free memory.

This file is collected last on purpose (it runs after the other GPU tests, and
it also passes alone in a fresh process)."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import (Batch, Engine, RkvError, noalloc_check_status,
                                           score_noalloc)
from decode_kv_cache_eviction_b200 import _binding as B
from oracle import rkv_oracle as ora

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ATOL, RTOL = 1e-6, 1e-3


def _batch(lengths, G, w, seed):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(off[-1])
    K = rng.standard_normal((T, 128)).astype(np.float32)
    K[rng.random(T) < 0.2] = K[0]                      # repeated keys
    Q = rng.standard_normal((len(lengths), G, w, 128)).astype(np.float32)
    t = lambda x: torch.from_numpy(x).to(DEV).to(torch.bfloat16)
    return Batch(t(K), t(K), t(Q), off)


def _close(x, ref, what):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    bad = ~(np.abs(x - ref) <= ATOL + RTOL * np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} entries out of tolerance"


@pytest.mark.parametrize("G,w", [(1, 8), (2, 8), (4, 8)])   # G * w = 8, 16, 32
def test_noalloc_matches_engine_and_oracle_on_consecutive_calls(G, w):
    b = _batch([3000, 5000, 777, 9], G, w, seed=G)
    eng = Engine(G, w, b.num_units, b.num_tokens, redundancy="gemm")
    a0, r0 = eng.alloc_scores(b)
    m0 = torch.empty_like(a0)
    eng.score(b, a0, r0, m0)
    eng.check_status()
    a1 = torch.full_like(a0, float("nan"))
    r1 = torch.full_like(a0, float("nan"))
    m1 = torch.full_like(a0, float("nan"))
    score_noalloc(G, w, b, a1, r1, m1)   # first call: per-device set-up
    noalloc_check_status()
    free0 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        for t in (a1, r1, m1):
            t.fill_(float("nan"))
        score_noalloc(G, w, b, a1, r1, m1)
        torch.cuda.synchronize()
        noalloc_check_status()
        assert torch.cuda.mem_get_info()[0] == free0, "a call changed the free device memory"
        ga, gr, gm = (t.double().cpu().numpy() for t in (a1, r1, m1))
        _close(ga, a0.double().cpu().numpy(), f"call {call} a vs engine")
        _close(gr, r0.double().cpu().numpy(), f"call {call} r vs engine")
        _close(gm, m0.double().cpu().numpy(), f"call {call} m vs engine")
        for u in range(b.num_units):
            lo, hi = int(b.tok_off_host[u]), int(b.tok_off_host[u + 1])
            c = hi - lo - w
            if c <= 0:
                continue
            k = b.K[lo:hi].double().cpu().numpy()
            q = b.Q[u].double().cpu().numpy()
            _, a_o = ora.importance(q, k)
            m_o, r_o = ora.redundancy_mean_closed_form(k, w)
            _close(ga[lo:lo + c], a_o, f"call {call} unit {u} a vs oracle")
            _close(gr[lo:lo + c], r_o, f"call {call} unit {u} r vs oracle")
            _close(gm[lo:lo + c], m_o, f"call {call} unit {u} m vs oracle")
    eng.close()


def test_noalloc_rejects_batches_beyond_its_static_scratch():
    G, w = 1, 8
    too_many = _batch([16] * 4097, G, w, seed=2)
    a = torch.empty(too_many.num_tokens, dtype=torch.float32, device=DEV)
    with pytest.raises(RkvError) as ei:
        score_noalloc(G, w, too_many, a, a.clone())
    assert ei.value.code == B.RKV_ERR_CAPACITY
    long_batch = _batch([40000] * 27, G, w, seed=3)    # 1,080,000 rows > 2^20
    a = torch.empty(long_batch.num_tokens, dtype=torch.float32, device=DEV)
    with pytest.raises(RkvError) as ei:
        score_noalloc(G, w, long_batch, a, a.clone())
    assert ei.value.code == B.RKV_ERR_CAPACITY
    wide = _batch([100], 8, 8, seed=4)                  # G * w = 64 > 32
    a = torch.empty(wide.num_tokens, dtype=torch.float32, device=DEV)
    with pytest.raises(RkvError) as ei:
        score_noalloc(8, 8, wide, a, a.clone())
    assert ei.value.code == B.RKV_ERR_UNSUPPORTED
