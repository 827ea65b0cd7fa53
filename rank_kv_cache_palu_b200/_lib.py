"""ctypes loader for the in-tree libpalu.so.

The product path has exactly one implementation: the CUDA kernels behind this
library.  If the library is missing this module raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpalu.so")

c_int32, c_float, c_size_t, c_void_p, c_int = (ctypes.c_int32, ctypes.c_float, ctypes.c_size_t,
                                               ctypes.c_void_p, ctypes.c_int)


class PaluConfig(ctypes.Structure):
    """Mirror of ``palu_config`` in include/palu.h."""

    _fields_ = [
        ("num_heads", c_int32),
        ("head_dim", c_int32),
        ("group_size", c_int32),
        ("rank_k", c_int32),
        ("rank_v", c_int32),
        ("page_size", c_int32),
        ("rope_base", c_float),
        ("act_dtype", c_int32),
        ("latent_dtype", c_int32),
    ]


_P = ctypes.POINTER
_CFG = _P(PaluConfig)

# name -> (restype, argtypes); one line per entry point of include/palu.h
SIGNATURES = {
    "palu_cache_strides": (c_int, [_CFG, _P(c_size_t), _P(c_size_t), _P(c_size_t), _P(c_size_t)]),
    "palu_compress_workspace_size": (c_int, [_CFG, c_int, c_int, _P(c_size_t)]),
    "palu_compress_append": (c_int, [_CFG, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_int, c_void_p, c_size_t, c_void_p]),
    "palu_decode_num_splits": (c_int, [_CFG, c_int, c_int, _P(c_int)]),
    "palu_decode_workspace_size": (c_int, [_CFG, c_int, c_int, c_int, _P(c_size_t)]),
    "palu_decode_multi_workspace_size": (c_int, [_CFG, c_int, c_int, c_int, c_int, _P(c_size_t)]),
    "palu_decode_attn_multi": (c_int, [_CFG, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p,
                                       c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_int,
                                       c_void_p]),
    "palu_decode_attn": (c_int, [_CFG, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_int, c_void_p]),
    "palu_decode_attn_noalloc": (c_int, [_CFG, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int,
                                         c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                         _P(c_int32)]),
    "palu_cache_strides_ranked": (c_int, [_CFG, _P(c_int32), _P(c_int32), _P(c_size_t), _P(c_size_t),
                                          _P(c_size_t), _P(c_size_t), _P(c_size_t), _P(c_size_t)]),
    "palu_compress_ranked_workspace_size": (c_int, [_CFG, _P(c_int32), _P(c_int32), c_int, c_int,
                                                    _P(c_size_t)]),
    "palu_compress_append_ranked": (c_int, [_CFG, _P(c_int32), _P(c_int32), c_int, c_int, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "palu_decode_ranked_workspace_size": (c_int, [_CFG, _P(c_int32), _P(c_int32), c_int, c_int, c_int, c_int,
                                                  _P(c_size_t)]),
    "palu_decode_attn_ranked": (c_int, [_CFG, _P(c_int32), _P(c_int32), c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                        c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                        c_size_t, c_int, c_void_p]),
    "palu_get_device_status": (c_int, [c_void_p, c_void_p, _P(c_int32)]),
    "palu_status_string": (ctypes.c_char_p, [c_int]),
    "palu_last_cuda_error": (ctypes.c_char_p, []),
    "palu_decode_kernel_kind": (c_int, [_CFG]),
    "palu_kernel_launches": (ctypes.c_uint64, []),
    "palu_debug_trace": (c_int, [c_void_p, c_size_t, c_int]),
    "palu_debug_timeout_test": (c_int, [ctypes.c_int64, c_int]),
}

_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load libpalu.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m rank_kv_cache_palu_b200.build` "
                    "(the CUDA kernels are the only implementation; there is no fallback)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib
