"""Error paths on the GPU without faulting it (failure detection).

Faults are injected on the host (rkv_inject_fault): an allocation that fails,
or one score chunk that never announces its statistics, so that the other
CTAs' bounded waits run out.  Each test checks the reported status and that
the engine (and the GPU context) work normally afterwards."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Engine, RkvError, inject_create_fault
from decode_kv_cache_eviction_b200 import _binding as B

from parity import check_unit, rand_batch, run_engine

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("mode", ["closed", "gemm"])
def test_dropped_announcement_times_out_then_engine_recovers(mode):
    lengths = [3000, 1500, 700]
    b = rand_batch(lengths, 4, 8, seed=21)
    eng = Engine(4, 8, len(lengths), b.num_tokens, redundancy=mode)
    a, r = eng.alloc_scores(b)
    eng.inject_fault(B.RKV_FAULT_DROP_ANNOUNCE)
    eng.score(b, a, r)
    with pytest.raises(RkvError) as ei:
        eng.check_status()
    assert ei.value.code == B.RKV_ERR_TIMEOUT
    eng.check_status()   # reading cleared the status word
    # the next call runs normally and matches the oracle
    out = run_engine(b, 4, 8, 0.1, 256, engine=eng)
    for u in range(len(lengths)):
        check_unit(out, b, u, 8, 0.1, 256)


def test_allocation_fault_in_adaptive_budget_then_recovers():
    b = rand_batch([2000, 900], 4, 8, seed=22)
    eng = Engine(4, 8, 2, b.num_tokens, redundancy="closed")
    p_last = torch.empty(b.num_tokens, dtype=torch.float32, device=DEV)
    budgets = torch.empty(2, dtype=torch.int32, device=DEV)
    eng.inject_fault(B.RKV_FAULT_ALLOC)
    with pytest.raises(RkvError) as ei:
        eng.refree_budget(b, 0.01, 4, 512, p_last, budgets)
    assert ei.value.code == B.RKV_ERR_OOM
    eng.refree_budget(b, 0.01, 4, 512, p_last, budgets)   # allocates now
    eng.check_status()
    assert torch.all(budgets >= 0)


def test_allocation_fault_in_host_pipeline_then_recovers():
    lengths = [1200, 800]
    b = rand_batch(lengths, 4, 8, seed=23)
    eng = Engine(4, 8, 2, b.num_tokens, redundancy="closed")
    K, V, Q = (t.cpu().pin_memory() for t in (b.K, b.V, b.Q))
    idx, nk, Ko, Vo = eng.alloc_host_outputs(2, 128)
    eng.inject_fault(B.RKV_FAULT_ALLOC)
    with pytest.raises(RkvError) as ei:
        eng.compress_host(K, V, Q, b.tok_off_host, 0.1, 128, idx, nk, Ko, Vo)
    assert ei.value.code == B.RKV_ERR_OOM
    eng.compress_host(K, V, Q, b.tok_off_host, 0.1, 128, idx, nk, Ko, Vo)
    eng.check_status()
    ref = run_engine(b, 4, 8, 0.1, 128, mode="closed")
    assert np.array_equal(idx.numpy(), ref["idx"]) and np.array_equal(nk.numpy(), ref["nk"])


def test_allocation_fault_at_creation_then_recovers():
    inject_create_fault(B.RKV_FAULT_ALLOC)
    with pytest.raises(RkvError) as ei:
        Engine(4, 8, 4, 10000, redundancy="gemm")
    assert ei.value.code == B.RKV_ERR_OOM
    eng = Engine(4, 8, 4, 10000, redundancy="gemm")
    b = rand_batch([2000], 4, 8, seed=24)
    out = run_engine(b, 4, 8, 0.1, 64, engine=eng)
    check_unit(out, b, 0, 8, 0.1, 64)
