"""ctypes declarations of libloki.so (the C ABI of include/loki.h).

Loading fails loudly: there is no CPU fallback.  Build the library with
``python -m sparse_decode_attention_loki_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libloki.so")

LOKI_OK = 0
LOKI_ERR_INVALID_ARG = 1
LOKI_ERR_UNSUPPORTED = 2
LOKI_ERR_CUDA = 3

LOKI_F32 = 0
LOKI_BF16 = 1


class loki_cache(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("k_hat", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("k_lr", ctypes.c_void_p),
        ("d_lr", ctypes.c_int32),
    ]


class loki_paged_cache(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("k_hat", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("k_lr", ctypes.c_void_p),
        ("d_lr", ctypes.c_int32),
    ]


class loki_seq_table(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("pages_per_seq", ctypes.c_int32),
        ("max_seq_len", ctypes.c_int32),
        ("block_table", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
    ]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_cache_p = ctypes.POINTER(loki_cache)
_pcache_p = ctypes.POINTER(loki_paged_cache)
_seqs_p = ctypes.POINTER(loki_seq_table)

# name -> (restype, argtypes); every entry point of include/loki.h
SIGNATURES = {
    "loki_append": (_i32, [_cache_p, _i32, _i32, _vp, _vp, _vp, _vp]),
    "loki_decode_workspace_size": (_i32, [_cache_p, _i32, _i32, ctypes.POINTER(ctypes.c_size_t)]),
    "loki_decode_attention": (_i32, [_cache_p, _i32, _i32, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp, _vp,
                                     ctypes.c_size_t, _vp]),
    "loki_decode_attention_noalloc": (_i32, [_cache_p, _i32, _i32, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp,
                                             _vp]),
    "dense_decode_attention": (_i32, [_cache_p, _i32, _i32, _vp, _vp, ctypes.c_float, _vp, _vp]),
    "loki_decode_attention_append": (_i32, [_cache_p, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _i32, ctypes.c_float,
                                            _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "dense_decode_attention_append": (_i32, [_cache_p, _i32, _i32, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp]),
    "loki_paged_decode_attention_append": (_i32, [_pcache_p, _seqs_p, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _i32,
                                                  ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "loki_topk_jaccard": (_i32, [_vp, _vp, _i32, _i32, _vp, _vp]),
    "loki_device_error_count": (_i32, [ctypes.POINTER(ctypes.c_uint32)]),
    "loki_decode_launch_shape": (_i32, [_cache_p, _i32, _i32, _i32, _i32, ctypes.POINTER(_i32)]),
    "loki_paged_append": (_i32, [_pcache_p, _seqs_p, _vp, _i32, _vp, _vp, _vp, _vp]),
    "loki_paged_decode_workspace_size": (_i32, [_pcache_p, _seqs_p, _i32, ctypes.POINTER(ctypes.c_size_t)]),
    "loki_paged_decode_attention": (_i32, [_pcache_p, _seqs_p, _i32, _vp, _vp, _i32, _vp, _i32, ctypes.c_float, _vp,
                                           _vp, _vp, ctypes.c_size_t, _vp]),
    "dense_paged_decode_attention": (_i32, [_pcache_p, _seqs_p, _i32, _vp, _vp, ctypes.c_float, _vp, _vp]),
    "loki_pca_workspace_size": (_i32, [_i32, _i32, ctypes.POINTER(ctypes.c_size_t)]),
    "loki_pca_calibrate": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "loki_set_launch_override": (_i32, [_i32]),
    "loki_phase_stamps": (_i32, [_i32, _i32, _vp, _i32, ctypes.POINTER(_i32)]),
    "loki_status_string": (ctypes.c_char_p, [_i32]),
    "loki_last_error": (ctypes.c_char_p, []),
    "loki_version": (_i32, []),
}

_lib = None


def load(path: str = None) -> ctypes.CDLL:
    """Load libloki.so once; raise if it is missing.  `path` (first call only)
    loads another build of the same library instead, e.g. one compiled with
    phase stamps."""
    global _lib
    if _lib is not None:
        if path is not None and path != _lib._name:
            raise RuntimeError(f"{_lib._name} is already loaded")
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m sparse_decode_attention_loki_b200.build` "
            "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class LokiError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} [{load().loki_status_string(status).decode()}]")
        self.status = status


def check(status: int) -> None:
    if status != LOKI_OK:
        raise LokiError(status, load().loki_last_error().decode())
