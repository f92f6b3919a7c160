"""bench.py's host-side arithmetic (CPU only): the algorithmic work per launch
that the roofline fractions divide by, the per-kernel report, and the
trigger-cadence workload."""
import types

import numpy as np

import bench
from decode_kv_cache_eviction_b200 import workloads as W


def fake_batch(lengths):
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return types.SimpleNamespace(tok_off_host=off, num_units=len(lengths),
                                 num_tokens=int(off[-1]))


def test_symmetric_gemm_tile_count():
    wl = W.custom(window=8, budget=64, group=4)
    lengths = [200, 512, 264, 32768, 8]
    alg = bench.algorithmic(fake_batch(lengths), wl)
    # tiles (a, b), a <= b, over ceil(N / 256) key blocks: 1, 3, 3 (the last
    # block of the 264-token unit holds window tokens only), 128 * 129 / 2; a
    # unit without candidates runs none
    tiles = 1 + 3 + 3 + 128 * 129 // 2
    assert alg["gemm_sym_flops"] == 2.0 * 128 * 256 * 256 * tiles
    n = np.array(lengths, dtype=np.float64)
    c = np.maximum(n - 8, 0)
    assert alg["gemm_flops"] == float((2 * c * n * 128).sum())
    # the symmetric form executes a bit more than half of the dense work at 32K
    one = bench.algorithmic(fake_batch([32768]), wl)
    assert 0.5 < one["gemm_sym_flops"] / one["gemm_flops"] < 0.51


def test_bytes_per_launch():
    wl = W.custom(window=8, budget=64, group=4)
    alg = bench.algorithmic(fake_batch([1000, 40]), wl)
    d, W_ = 128, 64 + 8
    assert alg["score_bytes"] == (2 * d + 8) * 1040 + 2 * d * 2 * 4 * 8
    assert alg["select_bytes"] == 8 * (992 + 32) + 4 * 2 * W_ + 4 * 2
    kept = min(992, 64) + 8 + min(32, 64) + 8
    assert alg["compact_bytes"] == 4 * d * kept + 4 * d * 2 * W_


def test_kernel_report_fractions():
    alg = {"gemm_flops": 2e12, "gemm_sym_flops": 1e12, "score_bytes": 6.5e9,
           "select_bytes": 1.3e9, "compact_bytes": 0.0, "evict_bytes": 0.0,
           "refree_bytes": 0.0}
    pk = {"hbm_gbs": 6500.0, "bf16_tflops_sustained": 1000.0}
    # (total ms, launches): 1 ms per launch
    rep = bench.kernel_report({"gemm": (2.0, 2), "score": (2.0, 2), "select": (0.5, 1),
                               "plan": (0.1, 0)}, alg, pk, "measured", symmetric=True)
    assert rep["gemm"]["achieved"] == 1000.0 and rep["gemm"]["frac"] == 1.0
    assert rep["gemm"]["dense_equivalent_tflops"] == 2000.0
    assert rep["score"]["achieved"] == 6500.0 and rep["score"]["frac"] == 1.0
    assert rep["select"]["frac"] == 0.4
    assert "plan" not in rep          # no launches: not reported
    dense = bench.kernel_report({"gemm": (1.0, 1)}, alg, pk, "measured", symmetric=False)
    assert dense["gemm"]["achieved"] == 2000.0 and "dense_equivalent_tflops" not in dense["gemm"]


def test_cadence_workload():
    wl = W.WORKLOADS["r1_llama8b_cadence"]
    every, trace = W.CADENCE[wl.name]
    assert wl.n_min == wl.n_max == wl.budget + every == 2176
    assert wl.num_units == 2048 and wl.group == 4 and wl.window == 8
    assert (trace - wl.budget) // every == 112
    assert wl.name not in W.WORKLOAD_ORDER and wl.name in W.EXTRA_WORKLOADS
