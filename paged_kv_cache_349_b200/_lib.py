"""ctypes loader for ``libpa.so`` (the CUDA library built from ``csrc/``).

There is no fallback: if the library cannot be loaded (or built with nvcc
when it is missing), importing the package fails.  ``PA_LIBRARY`` may name a
tuning build of the same sources to load instead.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_U64 = ctypes.c_uint64
_SZ = ctypes.c_size_t
_F = ctypes.c_float
_PI = ctypes.POINTER(ctypes.c_int)

# name -> (restype, argtypes); mirrors include/pa.h
SIGNATURES = {
    "pa_status_string": (ctypes.c_char_p, [_I]),
    "pa_version": (_I, []),
    "pa_launch_count": (_U64, []),
    "pa_reshape_and_cache": (_I, [_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _P, _P]),
    "pa_copy_blocks": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _P, _P]),
    "pa_swap_blocks": (_I, [_P, _P, _I64, _P, _P, _I64, _P, _I, _I, _I, _I, _P, _P]),
    "pa_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I]),
    "pa_decode_partition_tokens": (_I, [_I, _I, _I, _I, _I, _I, _I]),
    "pa_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _I, _P, _SZ, _P, _P]),
    "pa_decode_append": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _I, _P, _SZ, _P, _P]),
    "pa_decode_step_staging_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "pa_decode_step_host": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I64, _F,
                                 _I, _I, _P, _SZ, _P, _P]),
    "pa_decode_step_host_fp8": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I64,
                                     _F, _F, _F, _I, _I, _P, _SZ, _P, _P]),
    "pa_decode_shared_prefix_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "pa_decode_shared_prefix": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I64, _F,
                                     _I, _P, _SZ, _P, _P]),
    "pa_decode_step_plan_create": (_I, [_P, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I64,
                                        _F, _I, _I, _P, _SZ, _I, _F, _F, ctypes.POINTER(_P)]),
    "pa_decode_step_plan_run": (_I, [_P, _I, _I, _P, _P]),
    "pa_decode_step_plan_set_shared_prefix": (_I, [_P, _P, _I]),
    "pa_decode_step_staging_size_shared_prefix": (_SZ, [_I, _I, _I, _I, _I, _I, _I, _I, _I, _I]),
    "pa_decode_step_plan_destroy": (None, [_P]),
    "pa_decode_builtin_scratch": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _I, _P, _P]),
    "pa_quantize_fp8": (_I, [_P, _P, _I64, _F, _P]),
    "pa_reshape_and_cache_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I64, _I, _I, _I, _F, _F, _P, _P]),
    "pa_copy_blocks_fp8": (_I, [_P, _P, _P, _I, _I64, _I, _I, _I, _P, _P]),
    "pa_swap_blocks_fp8": (_I, [_P, _P, _I64, _P, _P, _I64, _P, _I, _I, _I, _I, _P, _P]),
    "pa_decode_fp8": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _F, _F, _I, _P, _SZ, _P,
                           _P]),
    "pa_decode_append_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I64, _F, _F, _F, _I,
                                  _P, _SZ, _P, _P]),
    "pa_alloc_create": (_I, [_I, _I, ctypes.POINTER(_P)]),
    "pa_alloc_create_ordered": (_I, [_I, _I, _P, ctypes.POINTER(_P)]),
    "pa_alloc_destroy": (None, [_P]),
    "pa_seq_create": (_I, [_P, _PI]),
    "pa_seq_append": (_I, [_P, _I, _P, _P, _P]),
    "pa_seq_append_batch": (_I, [_P, _P, _I, _P, _P, _PI]),
    "pa_seq_fork": (_I, [_P, _I, _PI]),
    "pa_seq_free": (_I, [_P, _I]),
    "pa_seq_block_table": (_I, [_P, _I, _P, _I, _PI, _PI]),
    "pa_alloc_export": (_I, [_P, _P, _I, _P, _I, ctypes.c_int32, _P]),
    "pa_alloc_step": (_I, [_P, _P, _I, _P, _I, ctypes.c_int32, _P, _P, _PI, _PI]),
    "pa_alloc_num_free": (_I, [_P]),
    "pa_validate_tables": (_I, [_P, _I, _I, _P, _I64, _I, _PI, _PI]),
    "pa_block_refcount": (_I, [_P, ctypes.c_int32]),
}


def load() -> ctypes.CDLL:
    """Load libpa.so (building it if missing).  PA_LIBRARY may name a tuning build
    of the same sources (build.py --define ... --out PATH) to load instead."""
    path = os.environ.get("PA_LIBRARY") or _build.LIB
    if path == _build.LIB and not os.path.exists(path):
        _build.build()
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()
