"""B200-native (sm_100a) engine for decode-time KV-cache compression, following
the R-KV method: importance + redundancy scoring, joint top-B eviction and
gather compaction, behind a small C ABI (``include/rkv.h``).

``Engine`` and ``Batch`` are a thin ctypes binding of ``librkv.so``; every step
runs in the library's CUDA kernels.
"""
from ._binding import (Batch, Engine, EXPORTS, LIB_PATH, RkvError, lib,  # noqa: F401
                       inject_create_fault, noalloc_check_status, score_noalloc, status_string)
