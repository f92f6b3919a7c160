"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function that include/rkv.h declares, its structs match the header byte
for byte, and argument validation rejects bad configurations before touching
the device."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

import decode_kv_cache_eviction_b200 as rkv
from decode_kv_cache_eviction_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rkv.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    from decode_kv_cache_eviction_b200 import build
    build.build()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rkv_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert header_functions() == sorted(B.EXPORTS)


def test_kernel_timing_ids_match_header():
    """The binding's per-kernel timing names are the header's RKV_KERNEL_*
    enum, in value order, and RKV_NUM_KERNELS counts them."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    ids = {m.group(1).lower(): int(m.group(2))
           for m in re.finditer(r"\bRKV_KERNEL_([A-Z]+)\s*=\s*(\d+)", text)}
    num = int(re.search(r"\bRKV_NUM_KERNELS\s*=\s*(\d+)", text).group(1))
    assert sorted(ids.values()) == list(range(num))
    assert tuple(sorted(ids, key=ids.get)) == B.KERNELS


def test_library_exports_every_header_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (rkv_\w+)", out))
    missing = set(header_functions()) - exported
    assert not missing, missing
    L = rkv.lib()
    for name in header_functions():
        assert getattr(L, name) is not None


def test_struct_layout_matches_header():
    src = r"""
    #include <stdio.h>
    #include <stddef.h>
    #include "rkv.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu %zu\n", sizeof(rkv_config), offsetof(rkv_config, max_tokens),
             offsetof(rkv_config, redundancy), offsetof(rkv_config, flags),
             offsetof(rkv_config, max_unit_tokens), sizeof(rkv_batch));
      printf("%zu %zu %zu %zu %zu\n", offsetof(rkv_batch, tok_off),
             offsetof(rkv_batch, tok_off_host), offsetof(rkv_batch, K),
             offsetof(rkv_batch, V), offsetof(rkv_batch, Q));
      printf("%zu %zu %zu %zu %zu\n", sizeof(rkv_host_batch), offsetof(rkv_host_batch, tok_off),
             offsetof(rkv_host_batch, K), offsetof(rkv_host_batch, V),
             offsetof(rkv_host_batch, Q));
      return 0;
    }
    """
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                        c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    want1 = [int(x) for x in lines[0].split()]
    want2 = [int(x) for x in lines[1].split()]
    C, Bt = B.RkvConfig, B.RkvBatch
    assert want1 == [ctypes.sizeof(C), C.max_tokens.offset, C.redundancy.offset,
                     C.flags.offset, C.max_unit_tokens.offset, ctypes.sizeof(Bt)]
    assert want2 == [Bt.tok_off.offset, Bt.tok_off_host.offset, Bt.K.offset, Bt.V.offset,
                     Bt.Q.offset]
    H = B.RkvHostBatch
    want3 = [int(x) for x in lines[2].split()]
    assert want3 == [ctypes.sizeof(H), H.tok_off.offset, H.K.offset, H.V.offset, H.Q.offset]


def test_status_strings_and_version():
    L = rkv.lib()
    assert L.rkv_version() == 10000
    for code in range(-7, 1):
        s = rkv.status_string(code)
        assert s and s != "unknown status"
    assert rkv.status_string(-99) == "unknown status"


def _create(**over):
    cfg = dict(head_dim=128, group=4, window=8, max_units=8, max_tokens=1 << 16,
               redundancy=0, flags=0)
    cfg.update(over)
    c = B.RkvConfig(**cfg)
    h = ctypes.c_void_p()
    return rkv.lib().rkv_create(ctypes.byref(c), ctypes.byref(h)), h


@pytest.mark.parametrize("over,code", [
    (dict(group=0), B.RKV_ERR_INVALID_ARG),
    (dict(window=0), B.RKV_ERR_INVALID_ARG),
    (dict(max_units=0), B.RKV_ERR_INVALID_ARG),
    (dict(max_tokens=0), B.RKV_ERR_INVALID_ARG),
    (dict(redundancy=7), B.RKV_ERR_INVALID_ARG),
    (dict(flags=8), B.RKV_ERR_INVALID_ARG),
    (dict(head_dim=64), B.RKV_ERR_UNSUPPORTED),
    (dict(group=16, window=17), B.RKV_ERR_UNSUPPORTED),   # G * w = 272 > 256
    (dict(max_unit_tokens=-1), B.RKV_ERR_INVALID_ARG),
    (dict(max_tokens=1 << 31), B.RKV_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config(over, code):
    rc, h = _create(**over)
    assert rc == code
    assert not h.value


def test_null_arguments():
    L = rkv.lib()
    h = ctypes.c_void_p()
    assert L.rkv_create(None, ctypes.byref(h)) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_score(None, None, None, None, None, None) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_select(None, None, None, None, 0.1, 4, None, None, None) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_compact(None, None, None, None, 4, None, None, None) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_check_status(None, None) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_compress_host(None, None, 0.1, 4, None, None, None, None, 0,
                               None) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_destroy(None) == B.RKV_OK
    assert L.rkv_launch_count(None) == 0


def test_fault_injection_arguments():
    L = rkv.lib()
    assert L.rkv_inject_fault(None, 7) == B.RKV_ERR_INVALID_ARG
    # dropping an announcement needs an engine (it concerns a score launch)
    assert L.rkv_inject_fault(None, B.RKV_FAULT_DROP_ANNOUNCE) == B.RKV_ERR_INVALID_ARG
    assert L.rkv_inject_fault(None, B.RKV_FAULT_ALLOC) == B.RKV_OK
    assert L.rkv_inject_fault(None, B.RKV_FAULT_NONE) == B.RKV_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU path")
def test_create_without_gpu_reports_cuda_error():
    rc, h = _create()
    assert rc in (B.RKV_ERR_CUDA, B.RKV_ERR_UNSUPPORTED)
    assert not h.value


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()
