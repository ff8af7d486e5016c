"""ctypes loader for the in-tree C-ABI library ``libfa_b200.so``.

The library is built by ``python -m exact_tiled_attention_42_b200.build``.
There is no fallback: if the library is missing, loading raises.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

_c_void_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_float = ctypes.c_float
_c_size_t = ctypes.c_size_t
_c_uint64 = ctypes.c_uint64

# name -> (restype, argtypes); mirrors include/fa.h
SIGNATURES = {
    "fa_fwd": (_c_int, [_c_void_p] * 5 + [_c_int] * 6 + [_c_float, _c_void_p]),
    "fa_bwd_workspace_size": (_c_size_t, [_c_int] * 5),
    "fa_bwd": (_c_int, [_c_void_p] * 10 + [_c_size_t] + [_c_int] * 6 + [_c_float, _c_void_p]),
    "fa_bwd_noalloc": (_c_int, [_c_void_p] * 9 + [_c_int] * 6 + [_c_float, _c_void_p]),
    "fa_fp8_workspace_size": (_c_size_t, [_c_int] * 5),
    "fa_fwd_fp8": (_c_int, [_c_void_p] * 5 + [_c_uint64, _c_int, _c_void_p, _c_size_t] + [_c_int] * 6
                   + [_c_float, _c_void_p]),
    "fa_mxfp8_workspace_size": (_c_size_t, [_c_int] * 5),
    "fa_fwd_mxfp8": (_c_int, [_c_void_p] * 5 + [_c_uint64, _c_int, _c_int, _c_void_p, _c_size_t] + [_c_int] * 6
                     + [_c_float, _c_void_p]),
    "fa_decode_workspace_size": (_c_size_t, [_c_int] * 7),
    "fa_fp8_quantize": (_c_int, [_c_void_p] * 3 + [_c_uint64, _c_int, _c_void_p, _c_size_t] + [_c_int] * 5 + [_c_void_p]),
    "fa_fwd_fp8_quantized": (_c_int, [_c_void_p, _c_size_t, _c_void_p, _c_void_p] + [_c_int] * 7 + [_c_float, _c_void_p]),
    "fa_fwd_decode": (_c_int, [_c_void_p] * 6 + [_c_size_t] + [_c_int] * 7 + [_c_float, _c_int, _c_void_p]),
    "fa_fwd_varlen": (_c_int, [_c_void_p] * 6 + [_c_int] * 7 + [_c_float, _c_void_p]),
    "fa_bwd_varlen_workspace_size": (_c_size_t, [_c_int] * 6),
    "fa_bwd_varlen": (_c_int, [_c_void_p] * 11 + [_c_size_t] + [_c_int] * 7 + [_c_float, _c_void_p]),
    "fa_status_string": (ctypes.c_char_p, [_c_int]),
    "fa_last_device_status": (_c_int, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load (once) and return the library with every signature declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m exact_tiled_attention_42_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
