#!/usr/bin/env python
"""Throughput of the decode-time KV-cache compression path (R-KV: importance +
redundancy scoring, joint top-B eviction, gather compaction) on B200.

One *step* = one rkv_compress call over the whole batch (score -> [plan ->
redundancy GEMM] -> select -> compact), inputs resident in HBM.  The metric is
KV tokens scored and evicted per second: sum over units of N_u, divided by the
step time.  Prints one JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl engine|reference]

Multi-GPU (torchrun): every rank compresses its own full batch (units are
independent: no collective on the data path); the step time is the maximum over
ranks, and `value` counts the tokens of all ranks ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_kv_cache_eviction_b200 import Batch, Engine, workloads as W  # noqa: E402

METRIC = "KV tokens scored+evicted/sec on 1 B200; % of HBM / tensor-core roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per launch of a kernel on long_trace_32k, from one
# ncu capture of a 16- or 64-unit profiling case scaled to 1024 units (traffic
# grows in proportion to the units processed).  Remove an entry whenever its
# kernel changes after the capture; the figures are in profiles/.
NCU_TRAFFIC_LONG_TRACE = {
    # (redundancy mode, kernel): bytes per launch
    ("gemm", "gemm"): (136.425472e6 + 5.207808e6) * 64,      # 16-unit capture
    ("gemm_sym", "gemm"): (137.337344e6 + 109.282048e6) * 64,  # 16-unit capture
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="engine", choices=["engine", "reference"])
    ap.add_argument("--workload", default="long_trace_32k",
                    choices=W.WORKLOAD_ORDER + W.EXTRA_WORKLOADS)
    ap.add_argument("--redundancy", default="gemm", choices=["gemm", "closed", "max"])
    ap.add_argument("--lam", type=float, default=0.1)
    ap.add_argument("--dense-gemm", dest="symmetric", action="store_false",
                    help="run the redundancy GEMM over all tiles instead of the symmetric form")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunk", type=int, default=0,
                    help="rows per chunk of the host-buffer pipeline (0: library default)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the second redundancy mode's measurement")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    return ap.parse_args()


# ---------------------------------------------------------------------- dist
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import torch.distributed as dist
            torch.cuda.set_device(self.local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


class _NoDist:
    rank, world, local = 0, 1, 0


# ---------------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv",
                                       "-i", str(index), "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.p = None

    def stop(self):
        if not self.p:
            return None
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        self.f.seek(0)
        rows = [ln.strip().split(", ") for ln in self.f.read().splitlines()[1:] if ln.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1].split()[0]))
                mx = float(r[2].split()[0])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip() == "Active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# oracle redundancy function that each engine mode computes
ORACLE_MODE = {"gemm": "rowblocks", "closed": "closed", "max": "max"}


def algorithmic(batch: Batch, wl: W.Workload):
    """Per-launch algorithmic work of each kernel (bytes or flops)."""
    n = np.diff(batch.tok_off_host).astype(np.float64)
    c = np.maximum(n - wl.window, 0)
    d = wl.head_dim
    kept = np.minimum(c, wl.budget) + np.minimum(n, wl.window)
    W_ = wl.budget + wl.window
    U = len(n)
    return {
        # K read once, a and r written
        "score_bytes": float((2 * d + 8) * n.sum() + 2 * d * U * wl.group * wl.window),
        # dense-equivalent tile products of the definition (rows in C x all N keys)
        "gemm_flops": float((2 * c * n * d).sum()),
        # symmetric form: the 256 x 256 tiles actually executed, (a, b) with
        # a <= b over the nb = ceil(N / 256) key blocks of a unit with candidates
        "gemm_sym_flops": float(sum(2 * d * 256 * 256 * (nb * (nb + 1) // 2)
                                    for nb, cc in zip(((n + 255) // 256).astype(np.int64), c)
                                    if cc > 0)),
        # a and r read, kept indices and counts written
        "select_bytes": float(8 * c.sum() + 4 * U * W_ + 4 * U),
        # kept K and V rows read; the whole [U, B+w] outputs written
        "compact_bytes": float(2 * 2 * d * kept.sum() + 2 * 2 * d * U * W_),
        # kept indices and counts read; keep mask (1 B) and free list (4 B) per
        # token and the free counts written
        "evict_bytes": float(4 * U * W_ + 4 * U + 5 * n.sum() + 4 * U),
        # K read once, the newest queries, p_last written and read back, budgets
        "refree_bytes": float((2 * d + 8) * n.sum() + 2 * d * U * wl.group + 8 * U),
        # symmetric form's finish: the partial-sum scratch (128 nb (nb + 3)
        # floats per unit with candidates) and rho read, m and r written
        "finish_bytes": float(sum(4 * 128 * nb * (nb + 3) + 12 * cc
                                  for nb, cc in zip(((n + 255) // 256).astype(np.int64), c)
                                  if cc > 0)),
    }


def timed(fn, steps, warmup, dist: Dist, eng=None):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    if eng is not None:
        eng.set_timing(True)
    l0 = eng.launches if eng is not None else 0
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    dist.barrier()
    ms = e0.elapsed_time(e1) / steps
    per_kernel = eng.read_timing() if eng is not None else {}
    launches = (eng.launches - l0) if eng is not None else 0
    if eng is not None:
        eng.set_timing(False)
    return dist.max(ms), per_kernel, launches


def kernel_report(per_kernel, alg, pk, src, symmetric=False):
    hbm = pk["hbm_gbs"]
    out = {}
    for name, (tot, n) in per_kernel.items():
        if n == 0:
            continue
        ms = tot / n
        ent = {"ms": round(ms, 4), "launches": n}
        if name == "gemm":
            # the tensor-pipe fraction counts the flops the kernel executes
            # (the symmetric form skips the tiles below the diagonal)
            flops = alg["gemm_sym_flops"] if symmetric else alg["gemm_flops"]
            tf = flops / (ms * 1e-3) / 1e12
            ent.update(bound="tensor", achieved=round(tf, 2), unit="TFLOP/s",
                       peak=pk["bf16_tflops_sustained"], frac=round(tf / pk["bf16_tflops_sustained"], 4))
            if symmetric:
                ent["dense_equivalent_tflops"] = round(alg["gemm_flops"] / (ms * 1e-3) / 1e12, 2)
        elif name in ("score", "select", "compact", "evict", "refree", "finish"):
            gbs = alg[f"{name}_bytes"] / (ms * 1e-3) / 1e9
            ent.update(bound="hbm", achieved=round(gbs, 1), unit="GB/s", peak=hbm,
                       frac=round(gbs / hbm, 4))
        ent["peak_source"] = src
        out[name] = ent
    return out


def cpu_baseline(batch: Batch, wl: W.Workload, lam: float, seconds: float, redundancy: str):
    """The fp64 oracle, as it stands, on a bounded sample of the same units."""
    from oracle import rkv_oracle as ora
    rng = np.random.default_rng(7)
    order = rng.permutation(batch.num_units)
    toks, t_used, done = 0, 0.0, 0
    mode = ORACLE_MODE[redundancy]
    for u in order:
        r0, r1 = int(batch.tok_off_host[u]), int(batch.tok_off_host[u + 1])
        k = batch.K[r0:r1].float().cpu().numpy().astype(np.float64)
        v = batch.V[r0:r1].float().cpu().numpy().astype(np.float64)
        q = batch.Q[u].float().cpu().numpy().astype(np.float64)
        t0 = time.perf_counter()
        ora.run_unit(q, k, v, wl.window, wl.budget, lam, redundancy=mode)
        t_used += time.perf_counter() - t0
        toks += r1 - r0
        done += 1
        if t_used >= seconds:
            break
    cores = len(os.sched_getaffinity(0))
    return {"value": toks / t_used, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": (f"{done} of {batch.num_units} units of {wl.name} "
                       f"(oracle.run_unit, {mode} redundancy, fp64 NumPy, "
                       f"{t_used:.1f} s on {cores} host threads)")}


def config_of(wl: W.Workload, batch: Batch, redundancy: str, lam: float, world: int,
              gemm_form: str = "dense"):
    n = np.diff(batch.tok_off_host)
    return {"workload": wl.name, "units": batch.num_units, "tokens": int(n.sum()),
            "n_min": int(n.min()), "n_max": int(n.max()), "head_dim": wl.head_dim,
            "group": wl.group, "window": wl.window, "budget": wl.budget, "lambda": lam,
            "redundancy": redundancy, "gemm": gemm_form,
            "l2": "inputs larger than L2 (K+V %.1f GiB per GPU)"
            % (2 * n.sum() * wl.head_dim * 2 / 2**30),
            "parallelism": f"replicas x{world} (units sharded per GPU, no collective)"}


# ---------------------------------------------------------------------- arms
def run_reference(args, dist: Dist):
    """The reference arm: the fp64 oracle on the host cores, one unit per step."""
    if dist.rank != 0:
        return
    from oracle import rkv_oracle as ora
    wl = W.WORKLOADS[args.workload]
    n = W.unit_lengths(wl, args.seed)
    rng = np.random.default_rng(11)
    units = rng.permutation(wl.num_units)[: args.steps + args.warmup]
    gb = W.generate(W.custom(name=wl.name, n_min=int(n[0]), n_max=int(n[0]), group=wl.group,
                             window=wl.window, budget=wl.budget, dup_frac=wl.dup_frac,
                             dup_noise=wl.dup_noise, span_len=wl.span_len,
                             key_scale=wl.key_scale, n_kv_head=len(units)),
                    seed=args.seed, device="cpu")
    mode = ORACLE_MODE[args.redundancy]
    times, toks = [], []
    for i in range(len(units)):
        r0, r1 = int(gb.tok_off[i]), int(gb.tok_off[i + 1])
        k = gb.K[r0:r1].float().numpy().astype(np.float64)
        v = gb.V[r0:r1].float().numpy().astype(np.float64)
        q = gb.Q[i].float().numpy().astype(np.float64)
        t0 = time.perf_counter()
        ora.run_unit(q, k, v, wl.window, wl.budget, args.lam, redundancy=mode)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            toks.append(r1 - r0)
    ms = 1e3 * sum(times) / len(times)
    value = sum(toks) / sum(times)
    cores = len(os.sched_getaffinity(0))
    sample = (f"one {wl.name}-shaped unit (N={int(n[0])}) per step, oracle.run_unit "
              f"({mode} redundancy, fp64 NumPy) on {cores} host threads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "redundancy": args.redundancy, "lambda": args.lam,
                       "sample": "one unit per step"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_engine(args, dist: Dist):
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    wl = W.WORKLOADS[args.workload]
    gb = W.generate(wl, seed=args.seed + dist.rank, device=dev)
    batch = Batch(gb.K, gb.V, gb.Q, gb.tok_off)
    tokens = batch.num_tokens
    pk, src = peaks()
    alg = algorithmic(batch, wl)

    def measure(mode):
        sym = mode == "gemm" and args.symmetric
        eng = Engine(wl.group, wl.window, batch.num_units, tokens, redundancy=mode,
                     symmetric_gemm=sym,
                     max_unit_tokens=int(np.diff(batch.tok_off_host).max()))
        a, r = eng.alloc_scores(batch)
        idx, nk, Ko, Vo = eng.alloc_outputs(batch, wl.budget)
        step = lambda: eng.compress(batch, args.lam, wl.budget, a, r, idx, nk, Ko, Vo)
        step()
        eng.check_status()
        ms, per_kernel, launches = timed(step, args.steps, args.warmup, dist, eng)
        eng.check_status()
        rep = kernel_report(per_kernel, alg, pk, src, symmetric=sym)
        del a, r, idx, nk, Ko, Vo
        return eng, ms, rep, launches

    clk = Clocks(dist.local) if dist.rank == 0 else None
    sym_main = args.redundancy == "gemm" and args.symmetric
    eng, ms, rep, launches = measure(args.redundancy)
    clocks = clk.stop() if clk else None
    value = tokens * dist.world / (ms * 1e-3)
    dom = "score" if args.redundancy == "closed" else "gemm"
    roof = dict(rep[dom])
    traffic = None
    if wl.name == "long_trace_32k":
        traffic = NCU_TRAFFIC_LONG_TRACE.get(("gemm_sym" if sym_main else args.redundancy, dom))
    roofline = {"kernel": dom, "bound": roof["bound"], "achieved": roof["achieved"],
                "peak": roof["peak"], "unit": roof["unit"], "frac": roof["frac"],
                "traffic": traffic, "traffic_unit": "bytes per launch (ncu, scaled)",
                "peak_source": ("%s (%s)" % (src, "bf16_tflops_sustained" if dom == "gemm"
                                              else "hbm_gbs"))}

    secondary = None
    if not args.no_secondary:
        other = "closed" if args.redundancy == "gemm" else "gemm"
        e2, ms2, rep2, _ = measure(other)
        e2.close()
        secondary = {"redundancy": other, "value": tokens * dist.world / (ms2 * 1e-3),
                     "ms_per_step": ms2, "kernels": rep2}

    in_place = adaptive = sweep = None
    if not args.no_secondary:
        in_place = measure_in_place(eng, batch, wl, args, dist, alg, pk, src)
        adaptive = measure_adaptive(eng, batch, wl, args, dist, alg, pk, src)
        if len(wl.lambdas) > 1:
            sweep = measure_lambda_sweep(eng, batch, wl, args, dist, alg, pk, src)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(eng, batch, wl, args, dist)
    eng.close()

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(batch, wl, args.lam, args.cpu_seconds, args.redundancy)

    if dist.rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": config_of(wl, batch, args.redundancy, args.lam, dist.world,
                                    "symmetric" if sym_main else "dense"),
                "roofline": roofline, "kernels": rep, "gpu_launches": launches,
                "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
                "secondary": secondary, "in_place": in_place, "adaptive": adaptive}
        if sweep is not None:
            line["lambda_sweep"] = sweep
        if wl.name in W.CADENCE:
            every, trace = W.CADENCE[wl.name]
            triggers = (trace - wl.budget) // every
            line["cadence"] = {"decode_steps_per_trigger": every, "trace_tokens": trace,
                               "triggers_per_trace": triggers, "ms_per_trigger": ms,
                               "ms_per_trace": ms * triggers}
        print(json.dumps(line), flush=True)


def measure_lambda_sweep(eng, batch: Batch, wl: W.Workload, args, dist: Dist, alg, pk, src):
    """The workload's lambda sweep: a and r do not depend on lambda, so one
    score serves every lambda, followed by select + compact per lambda.  The
    value counts each lambda's eviction of every token."""
    a, r = eng.alloc_scores(batch)
    outs = [eng.alloc_outputs(batch, wl.budget) for _ in wl.lambdas]

    def step():
        eng.score(batch, a, r)
        for lam, (idx, nk, Ko, Vo) in zip(wl.lambdas, outs):
            eng.select(batch, a, r, lam, wl.budget, idx, nk)
            eng.compact(batch, idx, nk, wl.budget, Ko, Vo)

    ms, per_kernel, _ = timed(step, args.steps, args.warmup, dist, eng)
    eng.check_status()
    rep = kernel_report(per_kernel, alg, pk, src)
    kept = [int(o[1].sum().item()) for o in outs]
    return {"lambdas": list(wl.lambdas),
            "value": batch.num_tokens * len(wl.lambdas) * dist.world / (ms * 1e-3),
            "ms_per_step": ms, "kept_tokens": kept,
            "kernels": {k: rep[k] for k in ("score", "select", "compact") if k in rep}}


def measure_adaptive(eng, batch: Batch, wl: W.Workload, args, dist: Dist, alg, pk, src):
    """The step with the adaptive budget: rkv_refree_budget (T = 1%, 4 sinks,
    budgets capped at the workload's B) -> score -> rkv_select_ex -> compact.
    The queries are scaled by 3 so that attention is peaked, as in a trained
    model; with the workload's unit-variance queries nearly every unit would
    need the whole cap and the budgets would not vary."""
    sinks, T, q_scale = 4, 0.01, 3.0
    batch = Batch(batch.K, batch.V, batch.Q * q_scale, batch.tok_off_host)
    a, r = eng.alloc_scores(batch)
    U, Wd = batch.num_units, wl.budget + sinks + wl.window
    dev = batch.K.device
    idx = torch.empty((U, Wd), dtype=torch.int32, device=dev)
    nk = torch.empty(U, dtype=torch.int32, device=dev)
    Ko = torch.empty((U, Wd, wl.head_dim), dtype=torch.bfloat16, device=dev)
    Vo = torch.empty_like(Ko)
    p_last = torch.empty(batch.num_tokens, device=dev)
    budgets = torch.empty(U, dtype=torch.int32, device=dev)

    def step():
        eng.refree_budget(batch, T, sinks, wl.budget, p_last, budgets)
        eng.score(batch, a, r)
        eng.select_ex(batch, a, r, args.lam, wl.budget, idx, nk, budgets, sinks)
        eng.compact(batch, idx, nk, wl.budget + sinks, Ko, Vo)

    ms, per_kernel, _ = timed(step, args.steps, args.warmup, dist, eng)
    eng.check_status()
    rep = kernel_report(per_kernel, alg, pk, src)
    b = budgets.cpu().numpy()
    return {"value": batch.num_tokens * dist.world / (ms * 1e-3), "ms_per_step": ms,
            "T": T, "sinks": sinks, "query_scale": q_scale, "budget_mean": float(b.mean()),
            "budget_min": int(b.min()), "budget_max": int(b.max()),
            "kernels": {k: rep[k] for k in ("refree", "select", "compact") if k in rep}}


def measure_in_place(eng, batch: Batch, wl: W.Workload, args, dist: Dist, alg, pk, src):
    """The same step with in-place slot reuse (rkv_evict_in_place: keep mask
    and free slots) in place of gather compaction."""
    a, r = eng.alloc_scores(batch)
    idx, nk = eng.alloc_outputs(batch, wl.budget)[:2]
    keep, free, nfree = eng.alloc_in_place(batch)

    def step():
        eng.score(batch, a, r)
        eng.select(batch, a, r, args.lam, wl.budget, idx, nk)
        eng.evict_in_place(batch, idx, nk, wl.budget, keep, free, nfree)

    ms, per_kernel, _ = timed(step, args.steps, args.warmup, dist, eng)
    eng.check_status()
    rep = kernel_report(per_kernel, alg, pk, src)
    return {"value": batch.num_tokens * dist.world / (ms * 1e-3), "ms_per_step": ms,
            "kernels": {k: rep[k] for k in ("select", "evict") if k in rep}}


def measure_e2e(eng, batch: Batch, wl: W.Workload, args, dist: Dist):
    """Same metric through the public host-buffer call (rkv_compress_host):
    page-locked host K, V, Q and offsets in, kept indices and compacted K/V out
    to page-locked host memory, the library's chunked copy-in / compute /
    copy-out pipeline inside the timed region."""
    hK = torch.empty(batch.K.shape, dtype=batch.K.dtype, pin_memory=True)
    hV = torch.empty(batch.V.shape, dtype=batch.V.dtype, pin_memory=True)
    hQ = torch.empty(batch.Q.shape, dtype=batch.Q.dtype, pin_memory=True)
    hK.copy_(batch.K)
    hV.copy_(batch.V)
    hQ.copy_(batch.Q)
    off = batch.tok_off_host
    outs = eng.alloc_host_outputs(batch.num_units, wl.budget)

    def step():
        eng.compress_host(hK, hV, hQ, off, args.lam, wl.budget, *outs,
                          chunk_tokens=args.e2e_chunk)

    ms, _, _ = timed(step, args.e2e_steps, 1, dist)
    eng.check_status()
    # the host path must reproduce the device path's kept indices exactly
    a, r = eng.alloc_scores(batch)
    idx, nk = eng.alloc_outputs(batch, wl.budget)[:2]
    eng.score(batch, a, r)
    eng.select(batch, a, r, args.lam, wl.budget, idx, nk)
    ok = torch.equal(outs[1], nk.cpu()) and torch.equal(outs[0], idx.cpu())
    # V crosses the bus whole only when it is not mapped into the device
    # address space; otherwise the compaction kernel reads the kept rows only
    v_mapped = _mapped_host(hV)
    v_bytes = (int(outs[1].sum()) * hV.shape[1] * hV.element_size() if v_mapped
               else hV.numel() * hV.element_size())
    h2d = sum(t.numel() * t.element_size() for t in (hK, hQ)) + v_bytes + 8 * len(off)
    d2h = sum(t.numel() * t.element_size() for t in outs)
    return {"value": batch.num_tokens * dist.world / (ms * 1e-3), "unit": UNIT,
            "ms_per_step": ms, "steps": args.e2e_steps, "warmup": 1,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "rkv_compress_host", "v_rows_moved": "kept" if v_mapped else "all",
            "outputs_consistent": bool(ok)}


def _mapped_host(t: torch.Tensor) -> bool:
    """Whether a host tensor is page-locked and visible to the device."""
    from cuda.bindings import runtime as rt
    err, attr = rt.cudaPointerGetAttributes(t.data_ptr())
    return (err == rt.cudaError_t.cudaSuccess and
            attr.type == rt.cudaMemoryType.cudaMemoryTypeHost and attr.devicePointer != 0)


def main():
    args = parse()
    if args.impl == "reference":
        # host-only arm: no process group; rank 0 alone runs, the others exit
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, _NoDist())
        return
    dist = Dist()
    try:
        run_engine(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
