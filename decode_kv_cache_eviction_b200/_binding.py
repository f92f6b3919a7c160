"""Thin ctypes binding of ``librkv.so`` (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module only turns
torch tensors into pointers and stream handles, checks dtypes and shapes, and
turns status codes into exceptions.  There is no fallback: if the library is
missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librkv.so")

RKV_OK = 0
RKV_ERR_INVALID_ARG = -1
RKV_ERR_UNSUPPORTED = -2
RKV_ERR_CUDA = -3
RKV_ERR_TIMEOUT = -4
RKV_ERR_OOM = -5
RKV_ERR_CAPACITY = -6
RKV_ERR_DEVICE = -7

RKV_REDUNDANCY_GEMM = 0
RKV_REDUNDANCY_CLOSED_FORM = 1
RKV_REDUNDANCY_MAX = 2
RKV_FLAG_GEMM_SINGLE_CTA = 1
RKV_FLAG_GEMM_SYMMETRIC = 2
RKV_FAULT_NONE = 0
RKV_FAULT_ALLOC = 1
RKV_FAULT_DROP_ANNOUNCE = 2

# Every function declared in include/rkv.h.
EXPORTS = ("rkv_create", "rkv_destroy", "rkv_score", "rkv_select", "rkv_compact",
           "rkv_compress", "rkv_compress_host", "rkv_evict_in_place", "rkv_fill_slots",
           "rkv_select_ex", "rkv_refree_budget", "rkv_check_status", "rkv_launch_count", "rkv_set_timing",
           "rkv_read_timing", "rkv_score_noalloc", "rkv_noalloc_check_status", "rkv_inject_fault",
           "rkv_debug_intermediates", "rkv_status_string", "rkv_version")
KERNELS = ("score", "plan", "gemm", "select", "compact", "evict", "fill", "refree", "finish")


class RkvConfig(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("group", ctypes.c_int),
                ("window", ctypes.c_int), ("max_units", ctypes.c_int),
                ("max_tokens", ctypes.c_int64), ("redundancy", ctypes.c_int),
                ("flags", ctypes.c_int), ("max_unit_tokens", ctypes.c_int64)]


class RkvHostBatch(ctypes.Structure):
    _fields_ = [("num_units", ctypes.c_int), ("tok_off", ctypes.c_void_p),
                ("K", ctypes.c_void_p), ("V", ctypes.c_void_p), ("Q", ctypes.c_void_p)]


class RkvBatch(ctypes.Structure):
    _fields_ = [("num_units", ctypes.c_int), ("tok_off", ctypes.c_void_p),
                ("tok_off_host", ctypes.c_void_p), ("K", ctypes.c_void_p),
                ("V", ctypes.c_void_p), ("Q", ctypes.c_void_p)]


class RkvError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


_lib = None


def lib():
    """Load ``librkv.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m decode_kv_cache_eviction_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    L.rkv_create.argtypes = [ctypes.POINTER(RkvConfig), ctypes.POINTER(vp)]
    L.rkv_destroy.argtypes = [vp]
    L.rkv_score.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, vp, vp]
    L.rkv_select.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, f32, i32, vp, vp, vp]
    L.rkv_compact.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, i32, vp, vp, vp]
    L.rkv_compress.argtypes = [vp, ctypes.POINTER(RkvBatch), f32, i32, vp, vp, vp, vp, vp,
                               vp, vp]
    L.rkv_compress_host.argtypes = [vp, ctypes.POINTER(RkvHostBatch), f32, i32, vp, vp, vp, vp,
                                    i64, vp]
    L.rkv_evict_in_place.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, i32, vp, vp, vp, vp]
    L.rkv_fill_slots.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, vp, vp, vp, vp, vp, vp,
                                 vp, vp]
    L.rkv_select_ex.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, f32, i32, vp, i32, vp, vp,
                                vp]
    L.rkv_refree_budget.argtypes = [vp, ctypes.POINTER(RkvBatch), f32, i32, i32, vp, vp, vp, vp]
    L.rkv_check_status.argtypes = [vp, vp]
    L.rkv_launch_count.argtypes = [vp]
    L.rkv_launch_count.restype = i64
    L.rkv_set_timing.argtypes = [vp, i32]
    L.rkv_read_timing.argtypes = [vp, i32, ctypes.POINTER(ctypes.c_double),
                                  ctypes.POINTER(i64)]
    L.rkv_score_noalloc.argtypes = [i32, i32, ctypes.POINTER(RkvBatch), vp, vp, vp, vp]
    L.rkv_noalloc_check_status.argtypes = [vp]
    L.rkv_inject_fault.argtypes = [vp, i32]
    L.rkv_debug_intermediates.argtypes = [vp, ctypes.POINTER(RkvBatch), vp, vp, vp]
    L.rkv_status_string.argtypes = [i32]
    L.rkv_status_string.restype = ctypes.c_char_p
    L.rkv_version.argtypes = []
    for name in ("rkv_create", "rkv_destroy", "rkv_score", "rkv_select", "rkv_compact",
                 "rkv_compress", "rkv_compress_host", "rkv_evict_in_place", "rkv_fill_slots",
                 "rkv_select_ex", "rkv_refree_budget", "rkv_check_status", "rkv_set_timing",
                 "rkv_read_timing",
                 "rkv_score_noalloc", "rkv_noalloc_check_status", "rkv_inject_fault",
                 "rkv_debug_intermediates", "rkv_version"):
        getattr(L, name).restype = i32
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().rkv_status_string(code).decode()


def _check(code: int, what: str):
    if code != RKV_OK:
        raise RkvError(code, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def score_noalloc(group: int, window: int, batch: "Batch", a, r, m=None, stream=None):
    """rkv_score_noalloc: GEMM-mode scores using only the library's static device
    scratch (no engine, no allocation by the library)."""
    _check(lib().rkv_score_noalloc(int(group), int(window), ctypes.byref(batch.c), _ptr(a),
                                   _ptr(r), _ptr(m), _stream(stream)), "rkv_score_noalloc")


def noalloc_check_status(stream=None):
    """rkv_noalloc_check_status: raise if a device wait of an rkv_score_noalloc
    call on the current device timed out since the last check (clears it)."""
    _check(lib().rkv_noalloc_check_status(_stream(stream)), "noalloc device status")


def inject_create_fault(fault: int):
    """rkv_inject_fault(NULL, fault): the next engine creation's workspace
    allocation fails (RKV_FAULT_ALLOC), for testing error paths."""
    _check(lib().rkv_inject_fault(None, int(fault)), "rkv_inject_fault")


class Batch:
    """Views of one batch of unit caches (tensors stay owned by the caller).

    K, V: [T, d] bf16 CUDA tensors; Q: [U, G, w, d] bf16; tok_off: host int64
    offsets [U+1] (a device copy is made once, here)."""

    def __init__(self, K, V, Q, tok_off):
        for name, t in (("K", K), ("V", V), ("Q", Q)):
            if t is not None:
                if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
                    raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
        self.K, self.V, self.Q = K, V, Q
        off = np.ascontiguousarray(np.asarray(tok_off, dtype=np.int64))
        self.tok_off_host = off
        dev = (K if K is not None else Q).device
        self.tok_off = torch.from_numpy(off).to(dev)
        self.c = RkvBatch(len(off) - 1, self.tok_off.data_ptr(),
                          off.ctypes.data, _ptr(K), _ptr(V), _ptr(Q))

    @property
    def num_units(self):
        return len(self.tok_off_host) - 1

    @property
    def num_tokens(self):
        return int(self.tok_off_host[-1])


class Engine:
    """One engine = one configuration and its device workspace.

    redundancy: "gemm" (K Kᵀ tiles on the tensor cores, row mean), "closed"
    (the same row mean in closed form, fused into the score kernel) or "max"
    (row max from the GEMM tiles).  single_cta_gemm: M = 128 MMAs on single
    CTAs instead of CTA pairs.  symmetric_gemm: with "gemm", only the tiles on
    and above the diagonal (RKV_FLAG_GEMM_SYMMETRIC; about half the MMAs, a
    partial-sum scratch of about N^2 / 128 bytes per unit, allocated here for
    max_tokens in units of max_unit_tokens).  max_unit_tokens: the longest unit
    a batch may hold (0: the engine's limit).
    """

    def __init__(self, group: int, window: int, max_units: int, max_tokens: int,
                 head_dim: int = 128, redundancy: str = "gemm", single_cta_gemm=False,
                 symmetric_gemm=False, max_unit_tokens: int = 0):
        mode = {"gemm": RKV_REDUNDANCY_GEMM, "closed": RKV_REDUNDANCY_CLOSED_FORM,
                "max": RKV_REDUNDANCY_MAX}[redundancy]
        flags = ((RKV_FLAG_GEMM_SINGLE_CTA if single_cta_gemm else 0) |
                 (RKV_FLAG_GEMM_SYMMETRIC if symmetric_gemm else 0))
        self.cfg = RkvConfig(head_dim, group, window, max_units, max_tokens, mode, flags,
                             max_unit_tokens)
        self.group, self.window = group, window
        h = ctypes.c_void_p()
        _check(lib().rkv_create(ctypes.byref(self.cfg), ctypes.byref(h)), "rkv_create")
        self.h = h

    def close(self):
        if getattr(self, "h", None):
            lib().rkv_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- calls ----------------------------------------------------------------
    def score(self, batch: Batch, a, r, m=None, stream=None):
        _check(lib().rkv_score(self.h, ctypes.byref(batch.c), _ptr(a), _ptr(r), _ptr(m),
                               _stream(stream)), "rkv_score")

    def select(self, batch: Batch, a, r, lam: float, budget: int, idx, n_kept, stream=None):
        _check(lib().rkv_select(self.h, ctypes.byref(batch.c), _ptr(a), _ptr(r),
                                float(lam), int(budget), _ptr(idx), _ptr(n_kept),
                                _stream(stream)), "rkv_select")

    def compact(self, batch: Batch, idx, n_kept, budget: int, K_out, V_out, stream=None):
        _check(lib().rkv_compact(self.h, ctypes.byref(batch.c), _ptr(idx), _ptr(n_kept),
                                 int(budget), _ptr(K_out), _ptr(V_out), _stream(stream)),
               "rkv_compact")

    def compress(self, batch: Batch, lam: float, budget: int, a, r, idx, n_kept, K_out,
                 V_out, stream=None):
        _check(lib().rkv_compress(self.h, ctypes.byref(batch.c), float(lam), int(budget),
                                  _ptr(a), _ptr(r), _ptr(idx), _ptr(n_kept), _ptr(K_out),
                                  _ptr(V_out), _stream(stream)), "rkv_compress")

    def compress_host(self, K, V, Q, tok_off, lam: float, budget: int, idx, n_kept, K_out,
                      V_out, chunk_tokens: int = 0, stream=None):
        """The whole path from host tensors to host tensors (``rkv_compress_host``).
        K, V [T, d], Q [U, G, w, d] bf16 and the outputs are CPU tensors (pinned for
        overlapped copies); ``tok_off`` is an int64 sequence of U + 1 row offsets.
        Outputs are complete once ``stream`` (default: torch's current) is synced."""
        for t in (K, V, Q, idx, n_kept, K_out, V_out):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("compress_host takes contiguous host tensors")
        off = np.ascontiguousarray(np.asarray(tok_off, dtype=np.int64))
        hb = RkvHostBatch(len(off) - 1, off.ctypes.data, K.data_ptr(), V.data_ptr(),
                          Q.data_ptr())
        _check(lib().rkv_compress_host(self.h, ctypes.byref(hb), float(lam), int(budget),
                                       _ptr(idx), _ptr(n_kept), _ptr(K_out), _ptr(V_out),
                                       int(chunk_tokens), _stream(stream)),
               "rkv_compress_host")

    def evict_in_place(self, batch: Batch, idx, n_kept, budget: int, keep, free_slots, n_free,
                       stream=None):
        """Keep mask and ascending free slots instead of compaction
        (``rkv_evict_in_place``); keep is uint8 [T], free_slots int32 [T],
        n_free int32 [U]."""
        _check(lib().rkv_evict_in_place(self.h, ctypes.byref(batch.c), _ptr(idx), _ptr(n_kept),
                                        int(budget), _ptr(keep), _ptr(free_slots), _ptr(n_free),
                                        _stream(stream)), "rkv_evict_in_place")

    def fill_slots(self, batch: Batch, new_off, K_new, V_new, keep, free_slots, n_free,
                   stream=None):
        """New tokens overwrite the lowest free slots of their unit
        (``rkv_fill_slots``), in place in batch.K / batch.V.  ``new_off`` is an
        int64 sequence of U + 1 row offsets into K_new / V_new."""
        off = np.ascontiguousarray(np.asarray(new_off, dtype=np.int64))
        dev = torch.from_numpy(off).to(batch.K.device)
        _check(lib().rkv_fill_slots(self.h, ctypes.byref(batch.c), _ptr(batch.K), _ptr(batch.V),
                                    _ptr(dev), off.ctypes.data, _ptr(K_new), _ptr(V_new),
                                    _ptr(keep), _ptr(free_slots), _ptr(n_free),
                                    _stream(stream)), "rkv_fill_slots")
        return dev   # keep the device offsets alive until the caller syncs

    def alloc_in_place(self, batch: Batch):
        """keep uint8 [T], free_slots int32 [T], n_free int32 [U] on the batch's device."""
        T, U, dev = batch.num_tokens, batch.num_units, batch.K.device
        return (torch.empty(T, dtype=torch.uint8, device=dev),
                torch.empty(T, dtype=torch.int32, device=dev),
                torch.empty(U, dtype=torch.int32, device=dev))

    def select_ex(self, batch: Batch, a, r, lam: float, budget: int, idx, n_kept, budgets=None,
                  sinks: int = 0, stream=None):
        """Selection with attention sinks and optional per-unit budgets
        (``rkv_select_ex``); idx has row stride budget + sinks + w."""
        _check(lib().rkv_select_ex(self.h, ctypes.byref(batch.c), _ptr(a), _ptr(r), float(lam),
                                   int(budget), _ptr(budgets), int(sinks), _ptr(idx),
                                   _ptr(n_kept), _stream(stream)), "rkv_select_ex")

    def refree_budget(self, batch: Batch, T: float, sinks: int, max_budget: int, p_last, budgets,
                      keep_count=None, stream=None):
        """Adaptive per-unit budgets from the newest query's attention row
        (``rkv_refree_budget``)."""
        _check(lib().rkv_refree_budget(self.h, ctypes.byref(batch.c), float(T), int(sinks),
                                       int(max_budget), _ptr(p_last), _ptr(budgets),
                                       _ptr(keep_count), _stream(stream)), "rkv_refree_budget")

    def check_status(self, stream=None):
        _check(lib().rkv_check_status(self.h, _stream(stream)), "device status")

    def inject_fault(self, fault: int):
        """Arm a one-shot fault (RKV_FAULT_*) for testing error paths."""
        _check(lib().rkv_inject_fault(self.h, int(fault)), "rkv_inject_fault")

    def debug_intermediates(self, batch: Batch, rho=None, U=None, stream=None):
        """rho [T] and/or U [U, 128] of the last score call on this batch
        (``rkv_debug_intermediates``)."""
        _check(lib().rkv_debug_intermediates(self.h, ctypes.byref(batch.c), _ptr(rho), _ptr(U),
                                             _stream(stream)), "rkv_debug_intermediates")

    def set_timing(self, enable: bool):
        _check(lib().rkv_set_timing(self.h, 1 if enable else 0), "rkv_set_timing")

    def read_timing(self):
        """{kernel: (total_ms, launches)} since the previous read."""
        out = {}
        for k, name in enumerate(KERNELS):
            ms, n = ctypes.c_double(), ctypes.c_int64()
            _check(lib().rkv_read_timing(self.h, k, ctypes.byref(ms), ctypes.byref(n)),
                   "rkv_read_timing")
            out[name] = (ms.value, n.value)
        lib().rkv_set_timing(self.h, 1)   # forget what was read
        return out

    @property
    def launches(self) -> int:
        return int(lib().rkv_launch_count(self.h))

    # -- allocation helpers (caller-owned outputs) ------------------------------
    def alloc_scores(self, batch: Batch):
        T = batch.num_tokens
        dev = batch.K.device
        return (torch.empty(T, dtype=torch.float32, device=dev),
                torch.empty(T, dtype=torch.float32, device=dev))

    def alloc_host_outputs(self, num_units: int, budget: int, pin: bool = True):
        """Host (page-locked unless ``pin`` is False) outputs for compress_host."""
        U, W = num_units, budget + self.window
        return (torch.empty((U, W), dtype=torch.int32, pin_memory=pin),
                torch.empty(U, dtype=torch.int32, pin_memory=pin),
                torch.empty((U, W, 128), dtype=torch.bfloat16, pin_memory=pin),
                torch.empty((U, W, 128), dtype=torch.bfloat16, pin_memory=pin))

    def alloc_outputs(self, batch: Batch, budget: int):
        U, W = batch.num_units, budget + self.window
        dev = batch.K.device
        return (torch.empty((U, W), dtype=torch.int32, device=dev),
                torch.empty(U, dtype=torch.int32, device=dev),
                torch.empty((U, W, 128), dtype=torch.bfloat16, device=dev),
                torch.empty((U, W, 128), dtype=torch.bfloat16, device=dev))
