"""Loads libfdllm.so (built in-tree) and declares the C ABI of include/fdllm.h.

There is no fallback: when the library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfdllm.so")

_c_int, _c_float, _c_size, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes); the order follows include/fdllm.h
SIGNATURES = {
    "fdllm_version": (_c_int, []),
    "fdllm_status_string": (ctypes.c_char_p, [_c_int]),
    "fdllm_fused_step_workspace_bytes": (_c_size, [_c_int] * 7),
    "fdllm_verify_step_workspace_bytes": (_c_size, [_c_int] * 8),
    "fdllm_accept_workspace_bytes": (_c_size, [_c_int] * 3),
    "fdllm_fused_step": (_c_int, [_c_int] * 7 + [_vp, _vp, _vp, _c_float, _vp, _vp, _vp, _vp,
                                                 _c_size, _vp]),
    "fdllm_fused_step_rows": (_c_int, [_c_int] * 7 + [_vp, _vp, _vp, _c_float, _vp, _vp, _vp,
                                                      _vp, _c_size, _vp]),
    "fdllm_qkv_rope_scatter": (_c_int, [_c_int] * 7 + [_vp, _vp, _vp, _c_float, _vp, _vp, _vp,
                                                       _vp, _c_size, _vp]),
    "fdllm_attend": (_c_int, [_c_int] * 6 + [_vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "fdllm_verify_step": (_c_int, [_c_int] * 8 + [_vp, _vp, _vp, _vp, _vp, _c_float, _vp, _vp,
                                                  _vp, _vp, _vp, _c_int, _vp, _c_size, _vp]),
    "fdllm_verify_qkv_rope_scatter": (_c_int, [_c_int] * 8 + [_vp, _vp, _vp, _vp, _c_float, _vp,
                                                              _vp, _vp, _vp, _vp, _vp, _c_size,
                                                              _vp]),
    "fdllm_verify_attend": (_c_int, [_c_int] * 7 + [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                                    _c_int, _vp, _c_size, _vp]),
    "fdllm_accept": (_c_int, [_c_int] * 3 + [_vp, _vp, _vp, _vp, _c_float, _c_float, _vp, _vp,
                                             _vp, _vp, _vp, _c_size, _vp]),
    "fdllm_accept_noalloc": (_c_int, [_c_int] * 3 + [_vp, _vp, _vp, _vp, _c_float, _c_float,
                                                     _vp, _vp, _vp, _vp, _vp]),
    "fdllm_track_select": (_c_int, [_c_int] * 6 + [_vp, _vp, _vp, _c_int, _vp, _vp, _vp, _c_size,
                                                    _vp]),
    "fdllm_attention_split": (_c_int, [_c_int] * 7 + [_vp]),
    "fdllm_bounded_wait_selftest": (_c_int, [ctypes.c_uint64, _vp, _c_size, _vp]),
    "fdllm_launch_count": (ctypes.c_uint64, []),
    "fdllm_get_status": (_c_int, [_vp, _vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once).  Raises ImportError if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python kv_cache_attention_fdllm_b200/build.py`"
                " (nvcc, sm_100a).  There is no CPU fallback.")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib
