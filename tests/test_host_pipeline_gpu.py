"""rkv_compress_host (host buffers in, host buffers out, chunked and pipelined)
against rkv_compress on device buffers: every kernel works per unit, so the
outputs must agree bit for bit however the units are cut into chunks."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import Engine, RkvError

from parity import check_unit, oracle_mode, rand_batch

pytestmark = pytest.mark.gpu

LENGTHS = [2500, 9, 700, 1800, 129, 4000, 300, 2999, 8, 1024]
G, WIN, LAM = 4, 8, 0.1


def device_reference(b, budget, mode):
    eng = Engine(G, WIN, max_units=b.num_units, max_tokens=b.num_tokens, redundancy=mode)
    a, r = eng.alloc_scores(b)
    outs = eng.alloc_outputs(b, budget)
    eng.compress(b, LAM, budget, a, r, *outs)
    eng.check_status()
    torch.cuda.synchronize()
    return dict(a=a.cpu().numpy(), r=r.cpu().numpy(), idx=outs[0].cpu().numpy(),
                nk=outs[1].cpu().numpy(), Ko=outs[2].cpu(), Vo=outs[3].cpu())


def host_inputs(b, pin=True):
    f = (lambda t: t.cpu().pin_memory()) if pin else (lambda t: t.cpu())
    return f(b.K), f(b.V), f(b.Q)


def run_host(eng, b, budget, chunk, pin=True):
    hK, hV, hQ = host_inputs(b, pin)
    outs = eng.alloc_host_outputs(b.num_units, budget, pin=pin)
    for t in outs:
        t.fill_(7)   # nothing may survive from before the call
    eng.compress_host(hK, hV, hQ, b.tok_off_host, LAM, budget, *outs, chunk_tokens=chunk)
    eng.check_status()
    torch.cuda.synchronize()
    return outs


def assert_same(ref, outs):
    idx, nk, Ko, Vo = outs
    assert np.array_equal(idx.numpy(), ref["idx"])
    assert np.array_equal(nk.numpy(), ref["nk"])
    assert torch.equal(Ko.view(torch.int16), ref["Ko"].view(torch.int16))
    assert torch.equal(Vo.view(torch.int16), ref["Vo"].view(torch.int16))


@pytest.mark.parametrize("mode", ["gemm", "closed", "max"])
@pytest.mark.parametrize("chunk", [0, 3000, 7000])
def test_host_pipeline_equals_device_path(mode, chunk):
    b = rand_batch(LENGTHS, G, WIN, seed=41)
    budget = 200
    ref = device_reference(b, budget, mode)
    eng = Engine(G, WIN, max_units=b.num_units, max_tokens=b.num_tokens, redundancy=mode)
    assert_same(ref, run_host(eng, b, budget, chunk))
    # and the kept sets agree with the oracle on a few units
    for u in (0, 5):
        check_unit(ref, b, u, WIN, LAM, budget, redundancy=oracle_mode(mode), check_m=False)


def test_pageable_buffers_and_repeated_calls():
    b = rand_batch(LENGTHS, G, WIN, seed=42)
    eng = Engine(G, WIN, max_units=b.num_units, max_tokens=b.num_tokens)
    for budget, chunk, pin in ((64, 3000, False), (300, 5000, True), (64, 0, True),
                               (1000, 9000, False)):
        ref = device_reference(b, budget, "gemm")
        assert_same(ref, run_host(eng, b, budget, chunk, pin=pin))


def test_batch_larger_than_engine_capacity():
    """Chunks are bounded by the engine's max_units / max_tokens, so a host batch
    may be larger than what the engine could take on the device in one call."""
    b = rand_batch(LENGTHS, G, WIN, seed=43)
    budget = 128
    ref = device_reference(b, budget, "gemm")
    small = Engine(G, WIN, max_units=3, max_tokens=5000)
    assert_same(ref, run_host(small, b, budget, 0))


def test_host_pipeline_rejections():
    b = rand_batch([3000, 200], G, WIN, seed=44)
    eng = Engine(G, WIN, max_units=2, max_tokens=2000)
    hK, hV, hQ = host_inputs(b)
    outs = eng.alloc_host_outputs(2, 64)
    with pytest.raises(RkvError) as ei:   # a unit longer than max_tokens
        eng.compress_host(hK, hV, hQ, b.tok_off_host, LAM, 64, *outs)
    assert ei.value.code == -6
    b2 = rand_batch([300, 200], G, WIN, seed=45)
    hK, hV, hQ = host_inputs(b2)
    outs = eng.alloc_host_outputs(2, 2500)
    with pytest.raises(RkvError) as ei:   # budget + w rows of output exceed max_tokens
        eng.compress_host(hK, hV, hQ, b2.tok_off_host, LAM, 2500, *outs)
    assert ei.value.code == -6
    with pytest.raises(RkvError) as ei:   # N < w
        eng.compress_host(hK, hV, hQ, np.array([0, 5, 500]), LAM, 64,
                          *eng.alloc_host_outputs(2, 64))
    assert ei.value.code == -1
    with pytest.raises(ValueError):       # device tensors are refused by the binding
        eng.compress_host(b2.K, b2.V, b2.Q, b2.tok_off_host, LAM, 64,
                          *eng.alloc_host_outputs(2, 64))
    # nothing was enqueued by the rejected calls: the engine still works
    ref = device_reference(b2, 64, "gemm")
    assert_same(ref, run_host(eng, b2, 64, 0))


def test_many_units_chunks_keep_the_batch_chunk_size():
    # 200 units: the whole batch scores in chunks of 8 tiles per CTA step,
    # while a 2-unit host chunk alone would use 1-tile chunks to fill the GPU
    lengths = [3000 + 13 * (i % 7) for i in range(200)]
    b = rand_batch(lengths, G, WIN, seed=47)
    ref = device_reference(b, 256, "closed")
    eng = Engine(G, WIN, max_units=b.num_units, max_tokens=b.num_tokens, redundancy="closed")
    for chunk in (0, 7000):
        assert_same(ref, run_host(eng, b, 256, chunk))
