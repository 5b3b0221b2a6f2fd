"""ctypes declarations of libpaged.so (the C ABI in include/paged.h).

The library is loaded from this package's directory only; if it is missing
the import of any op raises immediately (there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpaged.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_OOM, PA_ERR_CUDA, PA_ERR_BAD_TABLE = range(6)
PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2

STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_OOM",
                4: "PA_ERR_CUDA", 5: "PA_ERR_BAD_TABLE"}

# (name, restype, argtypes) of every exported call, in header order.
_P = ctypes.c_void_p
_i32, _i64, _f32, _sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_st = ctypes.c_int
SIGNATURES = [
    ("pa_last_error", ctypes.c_char_p, []),
    ("pa_reshape_and_cache", _st, [_P, _P, _P, _P, _P, _i32, _i32, _i32, _i32, _i64, _st, _st,
                                   _P, _P, _P]),
    ("pa_decode", _st, [_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32, _i32, _i32, _i64,
                        _f32, _st, _st, _P, _P, _i32, _P, _sz, _P]),
    ("pa_decode_noalloc", _st, [_P, _P, _P, _P, _P, _i32, _P, _i32, _i32, _i32, _i32, _i32,
                                _i32, _i64, _f32, _st, _st, _P, _P, _i32, _P]),
    ("pa_decode_noalloc_check", _st, [_P]),
    ("pa_chunked_prefill", _st, [_P, _P, _P, _i32, _i32, _P, _P, _P, _i32, _P, _i32, _i32,
                                 _i32, _i32, _i32, _i32, _i64, _f32, _st, _st, _P, _P, _P, _sz,
                                 _P]),
    ("pa_chunked_prefill_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _st]),
    ("pa_decode_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _st]),
    ("pa_decode_partition_tokens", _i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _st]),
    ("pa_decode_check", _st, [_P, _P]),
    ("pa_workspace_init", _st, [_P, _sz, _P]),
    ("pa_inject_wait_timeout", _st, [_i32, ctypes.c_uint64]),
    ("pa_copy_blocks", _st, [_P, _P, _P, _P, _P, _i32, _i64, _i64, _i64, _P, _P]),
    ("pa_sha256", _st, [_P, _i64, _P]),
    ("pa_block_hash", _st, [_P, _P, _i32, _P]),
    ("pa_prompt_block_hashes", _st, [_P, _i64, _i32, _P]),
    ("pa_alloc_create", _st, [_i64, _P, ctypes.POINTER(_P)]),
    ("pa_alloc_destroy", None, [_P]),
    ("pa_alloc_allocate", _st, [_P, _i32, _P]),
    ("pa_alloc_share", _st, [_P, _i32]),
    ("pa_alloc_free", _st, [_P, _P, _i32]),
    ("pa_alloc_copy_on_write", _st, [_P, _i32, ctypes.POINTER(_i32), ctypes.POINTER(_i32)]),
    ("pa_alloc_acquire_prefix", _st, [_P, _P, _i32, _P, ctypes.POINTER(_i32)]),
    ("pa_alloc_register_hash", _st, [_P, _i32, _P]),
    ("pa_alloc_lookup", _i32, [_P, _P]),
    ("pa_alloc_num_free", _i64, [_P]),
    ("pa_alloc_num_blocks", _i64, [_P]),
    ("pa_alloc_refcount", _i32, [_P, _i32]),
    ("pa_alloc_free_list", _i64, [_P, _P, _i64]),
    ("pa_build_block_table", _st, [_P, _P, _i32, _i32, _P]),
    ("pa_build_slot_mapping", _st, [_P, _i32, _i32, _P, _P, _i32, _i32, _P]),
]

_lock = threading.Lock()
_lib = None


class PagedError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libpaged.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"libpaged.so not found at {LIB_PATH}; build it with "
                    "`python -m paged_kv_cache_448_b200.build` (there is no CPU fallback)")
            h = ctypes.CDLL(LIB_PATH)
            for name, res, args in SIGNATURES:
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _lib = h
        return _lib


def check(status: int) -> None:
    if status != PA_OK:
        msg = lib().pa_last_error()
        raise PagedError(status, msg.decode() if msg else "")
