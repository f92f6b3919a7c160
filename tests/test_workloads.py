"""The synthetic workload generator produces the stated shapes and duplicate
structure (CPU only; small or single-unit cases)."""
import numpy as np
import pytest
import torch

from decode_kv_cache_eviction_b200 import workloads as W


def test_five_workloads_have_the_stated_shapes():
    t, l1, c2, c3, c4 = (W.WORKLOADS[n] for n in W.WORKLOAD_ORDER)
    assert (t.num_units, t.group, t.n_min, t.budget, t.window) == (1, 1, 1024, 256, 8)
    assert (l1.num_units, l1.group, l1.n_min, l1.budget) == (8, 4, 4096, 1024)
    assert (c2.num_units, c2.n_min, c2.budget) == (2048, 16384, 2048)
    assert (c3.num_units, c3.n_min, c3.budget) == (1024, 32768, 4096)
    assert (c4.num_units, c4.n_min, c4.n_max, c4.budget) == (16384, 2048, 8192, 1024)
    assert c4.lambdas == (0.0, 0.1, 1.0)
    # R1-Llama-8B cache bytes per token: 2 (K,V) * 32 layers * 8 heads * 128 * 2 B
    assert 2 * c3.n_layer * c3.n_kv_head * c3.head_dim * 2 == 128 * 1024


def test_ragged_lengths_shared_within_a_sequence():
    wl = W.WORKLOADS["ragged_serving"]
    n = W.unit_lengths(wl, 0)
    per = n.reshape(wl.n_seq, wl.n_layer * wl.n_kv_head)
    assert np.all(per == per[:, :1])
    assert per.min() >= 2048 and per.max() <= 8192
    assert len(np.unique(per[:, 0])) > 20
    off = W.token_offsets(wl, 0)
    assert off[0] == 0 and np.all(np.diff(off) == n)


def test_single_token_copies_point_backwards():
    wl = W.WORKLOADS["tiny"]
    src = W.copy_maps(wl, 3)[0]
    copies = np.nonzero(src != np.arange(len(src)))[0]
    assert abs(len(copies) - 0.2 * 1024) <= 2
    assert np.all(src[copies] < copies)
    assert np.all(src[src] == src)  # roots only


@pytest.mark.parametrize("name,lo,hi", [("llama3_8b_layer", 64, 64),
                                        ("long_trace_32k", 32, 256)])
def test_span_copies(name, lo, hi):
    wl = W.WORKLOADS[name]
    n = int(W.unit_lengths(wl, 0)[0])
    src = W.copy_maps(wl, 1, [0])[0]
    is_copy = src != np.arange(n)
    frac = is_copy.mean()
    assert wl.dup_frac - 0.01 <= frac <= wl.dup_frac + 0.01 + hi / n
    # contiguous destination runs have the stated lengths (adjacent spans may touch)
    edges = np.diff(np.concatenate([[0], is_copy.astype(np.int8), [0]]))
    runs = np.nonzero(edges == -1)[0] - np.nonzero(edges == 1)[0]
    assert runs.min() >= lo
    assert np.all(src[is_copy] < np.nonzero(is_copy)[0])


def test_generate_is_seeded_bf16_and_copies_are_close():
    wl = W.custom(n_min=600, dup_frac=0.25, dup_noise=0.05, group=2, window=4)
    b1 = W.generate(wl, seed=5)
    b2 = W.generate(wl, seed=5)
    assert torch.equal(b1.K, b2.K) and torch.equal(b1.Q, b2.Q)
    assert b1.K.dtype == torch.bfloat16 and b1.Q.shape == (1, 2, 4, 128)
    src = W.copy_maps(wl, 5)[0]
    cp = np.nonzero(src != np.arange(600))[0]
    K = b1.K.float().numpy()
    d = np.linalg.norm(K[cp] - K[src[cp]], axis=1)
    assert np.all(d < 0.05 * np.sqrt(128) * 2)   # noise only (bf16 rounding aside)
    other = np.linalg.norm(K[cp] - K[(src[cp] + 1) % 600], axis=1)
    assert np.all(other > 5)


def test_exact_duplicates_when_noise_is_zero():
    wl = W.custom(n_min=400, dup_frac=0.15, dup_noise=0.0)
    b = W.generate(wl, seed=2)
    src = W.copy_maps(wl, 2)[0]
    cp = np.nonzero(src != np.arange(400))[0]
    assert torch.equal(b.K[cp], b.K[src[cp]])


def test_key_scale_per_unit_channel():
    wl = W.custom(n_min=300, n_kv_head=2, dup_frac=0.0, key_scale=(0.5, 4.0))
    b = W.generate(wl, seed=0)
    std = b.K[:300].float().std(dim=0)
    assert std.min() > 0.3 and std.max() < 5.0 and std.max() / std.min() > 2.5
