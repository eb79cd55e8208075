"""ctypes loader for libpa.so: struct layouts and function signatures of
include/pa.h.  Argument marshalling only — every step of the hot path runs
in the library's CUDA kernels; there is no fallback."""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_uint32, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpa.so")


class PaTensor(ctypes.Structure):
    _fields_ = [
        ("data", c_void_p),
        ("dtype", c_int32),
        ("ndim", c_int32),
        ("shape", c_int64 * 5),
        ("stride", c_int64 * 5),
    ]


class PaOpts(ctypes.Structure):
    _fields_ = [
        ("stream", c_void_p),
        ("workspace", c_void_p),
        ("workspace_bytes", c_size_t),
        ("partition_tokens", c_int32),
        ("timeout_ms", c_int32),
    ]


class PaAllocStats(ctypes.Structure):
    _fields_ = [
        ("num_blocks", c_int32),
        ("num_free", c_int32),
        ("num_seqs", c_int32),
        ("block_size", c_int32),
        ("num_tokens", c_int64),
        ("waste_slots", c_int64),
        ("num_cached", c_int32),
        ("num_evictable", c_int32),
    ]


PA_OK = 0
STATUS_NAMES = {
    0: "PA_OK",
    1: "PA_ERR_INVALID_ARG",
    2: "PA_ERR_UNSUPPORTED",
    3: "PA_ERR_OUT_OF_BLOCKS",
    4: "PA_ERR_CUDA",
    5: "PA_ERR_DEVICE_TIMEOUT",
    6: "PA_ERR_DEVICE_BOUNDS",
    7: "PA_ERR_SCRATCH_LIMIT",
    8: "PA_ERR_HOST_ALLOC",
}
PA_F32, PA_BF16, PA_I32, PA_I64, PA_FP8_E4M3 = 0, 1, 2, 3, 4
PA_DEV_TIMEOUT, PA_DEV_BAD_BLOCK, PA_DEV_BAD_CONTEXT, PA_DEV_BAD_SLOT = 0x1, 0x2, 0x4, 0x8
PA_DEV_BAD_WORKSPACE = 0x10
PA_DECODE_WS_HEADER_BYTES = 64 * 1024

_T = POINTER(PaTensor)
_O = POINTER(PaOpts)
_A = c_void_p  # opaque pa_allocator*
_I64P = POINTER(c_int64)
_I32P = POINTER(c_int32)

SIGNATURES = {
    "pa_reshape_and_cache": (c_int32, [_T, _T, _T, _T, _T, _O]),
    "pa_copy_blocks": (c_int32, [_T, _T, _T, _O]),
    "pa_decode": (c_int32, [_T, _T, _T, _T, _T, _T, c_float, c_int32, _O]),
    "pa_decode_no_alloc": (c_int32, [_T, _T, _T, _T, _T, _T, c_float, c_int32, _O]),
    "pa_reshape_and_cache_fp8": (c_int32, [_T, _T, _T, _T, _T, _T, _T, _O]),
    "pa_decode_fp8": (c_int32, [_T, _T, _T, _T, _T, _T, c_float, c_int32, _T, _T, _O]),
    "pa_prefill": (c_int32, [_T, _T, _T, _T, _T, _T, _T, c_int32, c_float, c_int32, _O]),
    "pa_decode_workspace_bytes": (c_int32, [c_int32, c_int32, c_int32, c_int32, c_int32, c_int32, POINTER(c_size_t)]),
    "pa_decode_cascade": (c_int32, [_T, _T, _T, _T, _T, _T, _T, _T, c_int32, c_float, c_int32, _O]),
    "pa_decode_cascade_workspace_bytes": (c_int32, [c_int32, c_int32, c_int32, c_int32, c_int32, c_int32,
                                                    POINTER(c_size_t)]),
    "pa_alloc_prefix_groups": (c_int32, [_A, _I64P, c_int32, c_int32, _I32P, _I32P, _I32P]),
    "pa_set_decode_tuning": (c_int32, [c_int32, c_int32, c_int32]),
    "pa_alloc_create": (c_int32, [c_int32, c_int32, _I32P, POINTER(_A)]),
    "pa_alloc_destroy": (None, [_A]),
    "pa_seq_add": (c_int32, [_A, c_int64]),
    "pa_seq_append": (c_int32, [_A, c_int64, c_int32, _I64P, _I64P, _I32P]),
    "pa_seq_append_batch": (c_int32, [_A, _I64P, _I32P, c_int32, _I64P, _I64P, _I32P, _I32P]),
    "pa_seq_fork": (c_int32, [_A, c_int64, c_int64]),
    "pa_seq_add_prefix": (c_int32, [_A, c_int64, _I64P, c_int32, _I32P]),
    "pa_seq_append_tokens": (c_int32, [_A, c_int64, _I64P, c_int32, _I64P, _I64P, _I32P]),
    "pa_alloc_evictable": (c_int32, [_A, _I32P, c_int32, _I32P]),
    "pa_alloc_set_host_pool": (c_int32, [_A, c_int32, _I32P]),
    "pa_seq_swap_out": (c_int32, [_A, c_int64, _I64P, c_int32, _I32P]),
    "pa_seq_swap_in": (c_int32, [_A, c_int64, _I64P, c_int32, _I32P]),
    "pa_alloc_num_host_free": (c_int32, [_A]),
    "pa_seq_host_table": (c_int32, [_A, c_int64, _I32P, c_int32, _I32P]),
    "pa_swap_blocks": (c_int32, [_T, _T, _T, _T, _T, _O]),
    "pa_seq_free": (c_int32, [_A, c_int64]),
    "pa_seq_len": (c_int32, [_A, c_int64, _I32P]),
    "pa_seq_block_table": (c_int32, [_A, c_int64, _I32P, c_int32, _I32P]),
    "pa_alloc_block_tables": (c_int32, [_A, _I64P, c_int32, _I32P, c_int32, _I32P]),
    "pa_alloc_num_free": (c_int32, [_A]),
    "pa_block_refcount": (c_int32, [_A, c_int32]),
    "pa_alloc_get_stats": (c_int32, [_A, POINTER(PaAllocStats)]),
    "pa_get_device_status": (c_int32, [_O, POINTER(c_uint32)]),
    "pa_debug_wait_selftest": (c_int32, [_O]),
    "pa_status_string": (ctypes.c_char_p, [c_int32]),
    "pa_version": (c_int32, []),
}

_lib = None


def load():
    """Load libpa.so (raises if it is missing: there is no other path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python paged_kv_cache_351_b200/build.py` "
            "(the CUDA library is the only implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        try:
            fn = getattr(lib, name)
        except AttributeError as e:
            raise ImportError(f"{LIB_PATH} lacks {name}: rebuild it with "
                              "`python paged_kv_cache_351_b200/build.py`") from e
        fn.restype = res
        fn.argtypes = args
    if lib.pa_version() != 1:
        raise ImportError("libpa.so version mismatch")
    _lib = lib
    return lib
