"""ctypes declarations of libstaple.so (include/staple.h), one per entry point.

Argument marshalling only: every computation happens in the library's CUDA
kernels.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libstaple.so")

c_status = C.c_int
vp = C.c_void_p
i32 = C.c_int32
i64 = C.c_int64
u32 = C.c_uint32
sz = C.c_size_t
P = C.POINTER


class staple_trace_record(C.Structure):
    _fields_ = [("kernel", C.c_char * 40), ("ms", C.c_float)]


class staple_embed(C.Structure):
    _fields_ = [("mode", i32), ("flags", u32), ("base", vp), ("row_pitch", i64),
                ("index", vp), ("n_rows", i64)]


class staple_adamw(C.Structure):
    _fields_ = [("lr", C.c_float), ("beta1", C.c_float), ("beta2", C.c_float), ("eps", C.c_float),
                ("weight_decay", C.c_float), ("step", i32)]


# name -> (restype, argtypes); mirrors include/staple.h
SIGNATURES = {
    "staple_abi_version": (C.c_int, []),
    "staple_status_string": (C.c_char_p, [c_status]),
    "staple_context_create": (c_status, [C.c_int, P(vp)]),
    "staple_context_destroy": (c_status, [vp]),
    "staple_get_error": (c_status, [vp, vp, P(i32)]),
    "staple_set_wait_limit": (c_status, [vp, i64]),
    "staple_set_sm_reserve": (c_status, [vp, i32]),
    "staple_trace_enable": (c_status, [vp, C.c_int]),
    "staple_trace_read": (c_status, [vp, vp, i32, P(i32)]),
    "staple_table_register": (c_status, [vp, vp, sz, i64, i32, i32, C.c_int, u32, P(vp)]),
    "staple_table_unregister": (c_status, [vp]),
    "staple_cache_build": (c_status, [vp, vp, vp, C.c_double, vp, P(vp)]),
    "staple_cache_info": (c_status, [vp, P(i32), P(i32)]),
    "staple_cache_hot_ids": (c_status, [vp, vp]),
    "staple_cache_rows": (c_status, [vp, P(vp)]),
    "staple_cache_free": (c_status, [vp]),
    "staple_workspace_bytes": (sz, [i32, i32, i32, u32]),
    "staple_dedup": (c_status, [vp, vp, i32, i64, vp, vp, vp, vp, vp, vp]),
    "staple_gather_unique_rows": (c_status, [vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]),
    "staple_gather_rows": (c_status, [vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      vp, vp]),
    "staple_ffn_fwd": (c_status, [vp, C.c_int, i32, i32, i32, vp, P(staple_embed), vp, vp, vp,
                                  vp, vp, vp, vp, vp, sz, vp]),
    "staple_embed_bwd": (c_status, [vp, C.c_int, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                    vp, vp, vp, sz, vp]),
    "staple_ffn_bwd": (c_status, [vp, C.c_int, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                  vp, vp, vp, sz, vp]),
    "staple_embed_grad_to_host": (c_status, [vp, i32, i32, vp, vp, vp, vp, vp, vp, vp]),
    "staple_cache_refresh": (c_status, [vp, vp, vp, vp, vp, vp, vp]),
    "staple_gather_unique_rows_bulk": (c_status, [vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                                  vp, i32, i32, vp]),
    "staple_adamw_rows": (c_status, [vp, i64, C.c_int, i32, vp, i32, vp, i64, vp, vp, i64,
                                     P(staple_adamw), i32]),
    "staple_embed_grad": (c_status, [vp, C.c_int, i32, i32, i32, vp, i64, vp, vp, vp, vp, vp, vp,
                                     sz, vp]),
    "staple_embed_grad_static": (c_status, [C.c_int, i32, i32, vp, i64, vp, vp, vp, vp, vp]),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libstaple.so and declare every prototype.  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"libstaple.so not found at {path}: build it with "
            "`python -m token_indexed_sparse_staple_b200.build` (there is no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib
