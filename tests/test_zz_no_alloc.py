"""rkv_score_noalloc: scoring for callers that cannot allocate device memory.

Some callers own every byte of HBM through their own allocator (a serving stack
that reserves nearly all memory for its KV block pool up front) or load this
library as a plug-in that must not call cudaMalloc behind the host framework's
back; they cannot create an engine, whose workspace is allocated.  This call
gives them the GEMM-mode scores with the library's fixed static device scratch
instead.  It must agree with the engine path (same tolerance as every parity
test: 1e-6 absolute + 1e-3 relative) on consecutive calls, since every call
reuses the same static scratch.

This file is collected last on purpose (it runs after the other GPU tests, and
it also passes alone in a fresh process)."""
import ctypes

import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Batch, Engine, RkvError, score_noalloc
from decode_kv_cache_eviction_b200 import _binding as B

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
    x, ref = x.double().cpu().numpy(), ref.double().cpu().numpy()
    bad = ~(np.abs(x - ref) <= ATOL + RTOL * np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} entries out of tolerance"


def test_noalloc_matches_engine_on_consecutive_calls():
    G, w = 4, 8
    b = _batch([3000, 5000, 777, 9], G, w, seed=1)
    eng = Engine(G, w, b.num_units, b.num_tokens, redundancy="gemm")
    a0, r0 = eng.alloc_scores(b)
    m0 = torch.empty_like(a0)
    eng.score(b, a0, r0, m0)
    eng.check_status()
    for call in range(2):
        a1 = torch.full_like(a0, float("nan"))
        r1 = torch.full_like(a0, float("nan"))
        m1 = torch.full_like(a0, float("nan"))
        score_noalloc(G, w, b, a1, r1, m1)
        torch.cuda.synchronize()
        _close(a1, a0, f"call {call} a")
        _close(r1, r0, f"call {call} r")
        _close(m1, m0, f"call {call} m")
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
