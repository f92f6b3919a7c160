"""Small profiling case for ncu (python -m decode_kv_cache_eviction_b200.profile_case): a long_trace_32k-shaped batch (N = 32768,
G = 4, w = 8, B = 4096, 30% span duplicates) with --units units, compressed
--iters times.  With --select-only U the scores of those units are tiled over U
units (the full workload's concurrency without its K and V on the device) and
only the selection runs.  Used only as the target of the ncu commands recorded
under profiles/; it is not part of the library."""
import argparse
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))  # repo root

import torch  # noqa: E402

from decode_kv_cache_eviction_b200 import Batch, Engine, workloads as W  # noqa: E402

ap = argparse.ArgumentParser()
ap.add_argument("--units", type=int, default=32)
ap.add_argument("--n", type=int, default=32768)
ap.add_argument("--mode", default="gemm", choices=["gemm", "closed", "max"])
ap.add_argument("--iters", type=int, default=3)
ap.add_argument("--symmetric", action="store_true", help="symmetric redundancy GEMM")
ap.add_argument("--extras", action="store_true",
                help="also run the in-place eviction and the adaptive-budget kernels")
ap.add_argument("--select-only", type=int, default=0,
                help="tile the units' scores over this many units and run only the selection")
a = ap.parse_args()
wl = W.custom(name="long_trace_32k", n_kv_head=a.units, group=4, window=8, budget=4096,
              n_min=a.n, dup_frac=0.3, dup_noise=0.05, span_len=(32, 256))
gb = W.generate(wl, seed=0, device="cuda")
b = Batch(gb.K, gb.V, gb.Q, gb.tok_off)
eng = Engine(4, 8, b.num_units, b.num_tokens, redundancy=a.mode, symmetric_gemm=a.symmetric)
ra, rr = eng.alloc_scores(b)
if a.select_only:
    eng.score(b, ra, rr)
    U2, n = a.select_only, a.n
    off2 = torch.arange(U2 + 1, dtype=torch.int64) * n
    a2 = ra.view(a.units, n).repeat((U2 + a.units - 1) // a.units, 1)[:U2].reshape(-1).contiguous()
    r2 = rr.view(a.units, n).repeat((U2 + a.units - 1) // a.units, 1)[:U2].reshape(-1).contiguous()
    del gb, b, eng
    torch.cuda.empty_cache()
    b2 = Batch(None, None, torch.zeros((1, 1, 1, 128), dtype=torch.bfloat16, device="cuda"),
               off2.numpy())
    eng2 = Engine(4, 8, U2, U2 * n, redundancy="closed")
    idx = torch.empty((U2, 4096 + 8), dtype=torch.int32, device="cuda")
    nk = torch.empty(U2, dtype=torch.int32, device="cuda")
    for _ in range(a.iters + 2):
        eng2.select(b2, a2, r2, 0.1, 4096, idx, nk)
    eng2.check_status()
    torch.cuda.synchronize()
    sys.exit(0)
idx, nk, Ko, Vo = eng.alloc_outputs(b, 4096)
for _ in range(a.iters):
    eng.compress(b, 0.1, 4096, ra, rr, idx, nk, Ko, Vo)
if a.extras:
    keep, free, nfree = eng.alloc_in_place(b)
    p_last = torch.empty(b.num_tokens, device="cuda")
    budgets = torch.empty(b.num_units, dtype=torch.int32, device="cuda")
    for _ in range(a.iters):
        eng.evict_in_place(b, idx, nk, 4096, keep, free, nfree)
        eng.refree_budget(b, 0.01, 4, 4096, p_last, budgets)
eng.check_status()
torch.cuda.synchronize()
print("ok", b.num_units, b.num_tokens)
