"""ctypes loader of the CUDA library (lib/libsbattn.so) with the C ABI's
argument types.  There is no fallback: if the library is missing the import
of any entry point raises."""

from __future__ import annotations

import ctypes
import os


_c_int, _c_double, _c_float, _c_size, _c_void = ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes); mirrors include/sbattn.h
SIGNATURES = {
    "sbattn_strerror": (ctypes.c_char_p, [_c_int]),
    "sbattn_version": (_c_int, []),
    "sbattn_check_status": (_c_int, [_c_void, _c_void]),
    "sbattn_keep_count": (_c_int, [_c_int, _c_double, ctypes.POINTER(_c_int)]),
    "sbattn_select_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "sbattn_qk_norm_rope": (_c_int, [_c_void] * 8 + [_c_int] * 9 + [_c_float, _c_float, _c_void]),
    "sbattn_select_blocks": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_double,
                                      _c_void, _c_void, _c_int, _c_void, _c_void, _c_size, _c_void]),
    "sbattn_select_blocks_pooled": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_double,
                                             _c_void, _c_void, _c_int, _c_void, _c_void]),
    "sbattn_select_blocks_threshold": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_float,
                                                _c_void, _c_void, _c_int, _c_void, _c_void]),
    "sbattn_select_blocks_noalloc": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_double,
                                              _c_void, _c_void, _c_int, _c_void, _c_void]),
    "sbattn_forward": (_c_int, [_c_void, _c_void, _c_void, _c_void, _c_void, _c_int, _c_void,
                                _c_int, _c_int, _c_int, _c_int, _c_float, _c_void, _c_void]),
    "sbattn_forward_diag": (_c_int, [_c_void, _c_void, _c_void, _c_void, _c_void, _c_int, _c_void,
                                     _c_int, _c_int, _c_int, _c_int, _c_float, _c_void, ctypes.c_ulonglong, _c_int,
                                     _c_void]),
    "sbattn_adaln_modulate": (_c_int, [_c_void, _c_void, _c_void, _c_void, _c_int, _c_int, _c_int, _c_float,
                                       _c_void]),
    "sbattn_swiglu": (_c_int, [_c_void, _c_void, _c_void, ctypes.c_int64, _c_int, ctypes.c_int64, _c_void]),
}

_LIB = None


def lib_path() -> str:
    from .build import LIB_PATH

    return LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library {path} is missing: build it with "
                "`python -m block_sparse_attention_qk_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def strerror(code: int) -> str:
    return lib().sbattn_strerror(code).decode()
