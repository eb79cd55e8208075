"""Python binding of libpa.so — paged KV cache attention for B200 (sm_100a).

Thin wrappers with the C ABI's names (include/pa.h).  They only turn torch
tensors and numpy arrays into the ABI's plain pointers, shapes and strides;
all device work runs in the library's CUDA kernels.  PyTorch is used by
callers for device memory and streams.  A non-OK status raises
``PagedAttentionError``.  Each device call runs with the device that holds
its CUDA tensors made current (tensors on two devices are refused); when no
stream is given, that device's current torch stream is used.
"""

from __future__ import annotations

import contextlib
import ctypes
from typing import Optional, Sequence, Tuple

import numpy as np

from . import _lib
from ._lib import (PA_DECODE_WS_HEADER_BYTES, PA_DEV_BAD_BLOCK, PA_DEV_BAD_CONTEXT,  # noqa: F401
                   PA_DEV_BAD_SLOT, PA_DEV_BAD_WORKSPACE, PA_DEV_TIMEOUT, PaAllocStats, PaOpts, PaTensor)

__all__ = [
    "PagedAttentionError", "OutOfBlocksError", "pa_reshape_and_cache", "pa_copy_blocks", "pa_decode",
    "pa_decode_workspace_bytes", "pa_decode_no_alloc", "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_prefill",
    "pa_decode_cascade", "pa_decode_cascade_workspace_bytes", "PreparedCall", "prepare_reshape_and_cache",
    "prepare_decode", "prepare_decode_cascade", "prepare_reshape_and_cache_fp8", "prepare_decode_fp8",
    "pa_swap_blocks", "pa_set_decode_tuning", "pa_get_device_status", "pa_debug_wait_selftest",
    "Allocator", "library",
]

_lib_handle = _lib.load()


def library():
    """The loaded ctypes library (for tests of the raw ABI)."""
    return _lib_handle


class PagedAttentionError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib_handle.pa_status_string(status)
        super().__init__(f"{where}: {_lib.STATUS_NAMES.get(status, status)} ({msg.decode() if msg else ''})")


class OutOfBlocksError(PagedAttentionError):
    pass


def _check(st: int, where: str) -> None:
    if st != 0:
        if st == 3:
            raise OutOfBlocksError(st, where)
        raise PagedAttentionError(st, where)


def _dtype_code(t) -> int:
    import torch

    codes = {torch.float32: _lib.PA_F32, torch.bfloat16: _lib.PA_BF16, torch.int32: _lib.PA_I32,
             torch.int64: _lib.PA_I64, torch.float8_e4m3fn: _lib.PA_FP8_E4M3}
    if t.dtype not in codes:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return codes[t.dtype]


def _tensor(t) -> PaTensor:
    """torch.Tensor -> pa_tensor (pointer, dtype, shape, strides in elements)."""
    pt = PaTensor()
    pt.data = t.data_ptr() if t.numel() > 0 else (t.data_ptr() or None)
    pt.dtype = _dtype_code(t)
    if t.dim() > 5:
        raise ValueError("at most 5 dimensions")
    pt.ndim = t.dim()
    for k in range(t.dim()):
        pt.shape[k] = t.shape[k]
        pt.stride[k] = t.stride(k)
    return pt


def _stream_ptr(stream) -> Optional[int]:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream or None
    return stream.cuda_stream or None


def _device_index(tensors) -> Optional[int]:
    """The CUDA device that holds the call's CUDA tensors (None when none is
    on a CUDA device, e.g. pinned host pools only).  Tensors on two CUDA
    devices are refused: one launch runs on one device."""
    idx = None
    for t in tensors:
        d = getattr(t, "device", None)
        if getattr(d, "type", None) != "cuda":  # host tensors, None, numpy's "cpu"
            continue
        i = 0 if d.index is None else int(d.index)
        if idx is None:
            idx = i
        elif i != idx:
            raise ValueError(f"tensors on cuda:{idx} and cuda:{i} in one call")
    return idx


def _on_device(tensors):
    """The library launches on the current CUDA device: make it the one that
    holds the tensors for the duration of the call (no switch when it already
    is, which is the usual one-process-per-GPU case)."""
    idx = _device_index(tensors)
    if idx is None:
        return contextlib.nullcontext()
    import torch

    if idx == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(idx)


def _opts(stream=None, workspace=None, partition_tokens: int = 0, timeout_ms: int = 0) -> PaOpts:
    o = PaOpts()
    o.stream = _stream_ptr(stream)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    else:
        o.workspace = None
        o.workspace_bytes = 0
    o.partition_tokens = partition_tokens
    o.timeout_ms = timeout_ms
    return o


# ---------------------------------------------------------------------------
# device entry points
# ---------------------------------------------------------------------------

def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Write each token's K/V [T, H_kv, D] into its slot of the paged cache."""
    tk, tv, kc, vc, sm = (_tensor(x) for x in (key, value, k_cache, v_cache, slot_mapping))
    with _on_device((key, value, k_cache, v_cache, slot_mapping)):
        o = _opts(stream)
        _check(_lib_handle.pa_reshape_and_cache(ctypes.byref(tk), ctypes.byref(tv), ctypes.byref(kc),
                                                ctypes.byref(vc), ctypes.byref(sm), ctypes.byref(o)),
               "pa_reshape_and_cache")


def pa_copy_blocks(k_cache, v_cache, pairs, stream=None) -> None:
    """Copy whole blocks (K and V) for each (src, dst) row of the int64 [n, 2] device tensor."""
    kc, vc, pr = (_tensor(x) for x in (k_cache, v_cache, pairs))
    with _on_device((k_cache, v_cache, pairs)):
        o = _opts(stream)
        _check(_lib_handle.pa_copy_blocks(ctypes.byref(kc), ctypes.byref(vc), ctypes.byref(pr), ctypes.byref(o)),
               "pa_copy_blocks")


def pa_decode(out, query, k_cache, v_cache, block_tables, context_lens, scale: float, num_kv_heads: int,
              workspace=None, partition_tokens: int = 0, stream=None, timeout_ms: int = 0) -> None:
    """Paged decode attention; writes out [B, H, D].  ``partition_tokens``:
    0 = auto (balanced split when ``workspace`` is large enough), >0 = fixed
    partitions, -1 = no split."""
    to, tq, kc, vc, bt, cl = (_tensor(x) for x in (out, query, k_cache, v_cache, block_tables, context_lens))
    with _on_device((out, query, k_cache, v_cache, block_tables, context_lens, workspace)):
        o = _opts(stream, workspace, partition_tokens, timeout_ms)
        _check(_lib_handle.pa_decode(ctypes.byref(to), ctypes.byref(tq), ctypes.byref(kc), ctypes.byref(vc),
                                     ctypes.byref(bt), ctypes.byref(cl), ctypes.c_float(scale), int(num_kv_heads),
                                     ctypes.byref(o)), "pa_decode")


def pa_decode_cascade(out, query, k_cache, v_cache, block_tables, context_lens, group_start, group_blocks,
                      max_group_size: int, scale: float, num_kv_heads: int, workspace, partition_tokens: int = 0,
                      stream=None, timeout_ms: int = 0) -> None:
    """Shared-prefix decode: pa_decode's result, with each group's shared
    leading blocks (int32 device tensors ``group_start`` [n_groups + 1] and
    ``group_blocks`` [n_groups], e.g. from ``Allocator.prefix_groups``) read
    once for all of the group's members.  ``workspace``: at least
    ``pa_decode_cascade_workspace_bytes`` bytes, zero-filled before first use."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens, group_start, group_blocks)
    ts = [_tensor(x) for x in args]
    with _on_device(args + (workspace,)):
        o = _opts(stream, workspace, partition_tokens, timeout_ms)
        _check(_lib_handle.pa_decode_cascade(*[ctypes.byref(t) for t in ts], int(max_group_size), ctypes.c_float(scale),
                                             int(num_kv_heads), ctypes.byref(o)), "pa_decode_cascade")


def pa_decode_cascade_workspace_bytes(num_seqs: int, num_heads: int, num_kv_heads: int, head_size: int,
                                      max_group_size: int, partition_tokens: int = 0) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib_handle.pa_decode_cascade_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_size, max_group_size,
                                                         partition_tokens, ctypes.byref(n)),
           "pa_decode_cascade_workspace_bytes")
    return int(n.value)


def pa_prefill(out, query, k_cache, v_cache, block_tables, context_lens, query_start, max_query_len: int,
               scale: float, num_kv_heads: int, stream=None, timeout_ms: int = 0) -> None:
    """Multi-token (chunked-prefill) paged attention: writes out [T, H, D]
    for the new tokens of every sequence (rows query_start[i] ..
    query_start[i+1]), each attending causally over its sequence's cache."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens, query_start)
    ts = [_tensor(x) for x in args]
    with _on_device(args):
        o = _opts(stream, timeout_ms=timeout_ms)
        _check(_lib_handle.pa_prefill(*[ctypes.byref(t) for t in ts], int(max_query_len), ctypes.c_float(scale),
                                      int(num_kv_heads), ctypes.byref(o)), "pa_prefill")


def pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale, stream=None) -> None:
    """Quantizing cache write into an FP8 (torch.float8_e4m3fn) cache: each
    value is stored as the e4m3 code of value / scale[kv head]."""
    args = (key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale)
    ts = [_tensor(x) for x in args]
    with _on_device(args):
        o = _opts(stream)
        _check(_lib_handle.pa_reshape_and_cache_fp8(*[ctypes.byref(t) for t in ts], ctypes.byref(o)),
               "pa_reshape_and_cache_fp8")


def pa_decode_fp8(out, query, k_cache, v_cache, block_tables, context_lens, scale: float, num_kv_heads: int,
                  k_scale, v_scale, workspace=None, partition_tokens: int = 0, stream=None, timeout_ms: int = 0) -> None:
    """Paged decode over an FP8 cache with per-kv-head scales; bf16 query and output."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens)
    ts = [_tensor(x) for x in args]
    ks, vs = _tensor(k_scale), _tensor(v_scale)
    with _on_device(args + (k_scale, v_scale, workspace)):
        o = _opts(stream, workspace, partition_tokens, timeout_ms)
        _check(_lib_handle.pa_decode_fp8(*[ctypes.byref(t) for t in ts], ctypes.c_float(scale), int(num_kv_heads),
                                         ctypes.byref(ks), ctypes.byref(vs), ctypes.byref(o)), "pa_decode_fp8")


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, pairs, stream=None) -> None:
    """Copy whole blocks between a device pool and a pinned host pool (either
    direction) for each (src, dst) row of ``pairs``."""
    args = (src_k, src_v, dst_k, dst_v, pairs)
    ts = [_tensor(x) for x in args]
    with _on_device(args):
        o = _opts(stream)
        _check(_lib_handle.pa_swap_blocks(*[ctypes.byref(t) for t in ts], ctypes.byref(o)), "pa_swap_blocks")


NO_ALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def pa_decode_no_alloc(out, query, k_cache, v_cache, block_tables, context_lens, scale: float, num_kv_heads: int,
                       partition_tokens: int = 0, stream=None, timeout_ms: int = 0) -> None:
    """pa_decode for callers that cannot provide device scratch (a host
    framework that owns all device memory and gives plugins no scratch
    buffer, or a loop that must not call cudaMalloc, which can synchronise
    the device).  The split scratch is a fixed 16 MiB array inside the
    library; a call needing more raises PA_ERR_SCRATCH_LIMIT.  The first call
    on a device looks up that array's address, so make it before any stream
    capture.  Calls share the array: issue them on one stream."""
    to, tq, kc, vc, bt, cl = (_tensor(x) for x in (out, query, k_cache, v_cache, block_tables, context_lens))
    with _on_device((out, query, k_cache, v_cache, block_tables, context_lens)):
        o = _opts(stream, None, partition_tokens, timeout_ms)
        _check(_lib_handle.pa_decode_no_alloc(ctypes.byref(to), ctypes.byref(tq), ctypes.byref(kc), ctypes.byref(vc),
                                              ctypes.byref(bt), ctypes.byref(cl), ctypes.c_float(scale),
                                              int(num_kv_heads), ctypes.byref(o)), "pa_decode_no_alloc")


def pa_decode_workspace_bytes(num_seqs: int, num_heads: int, num_kv_heads: int, head_size: int,
                              max_blocks_per_seq: int, partition_tokens: int = 0) -> int:
    """Bytes of decode workspace for these sizes on the current device (0
    for no split).  A workspace must be zero-filled before its first use
    (its header holds merge counters that every call leaves at zero)."""
    n = ctypes.c_size_t(0)
    _check(_lib_handle.pa_decode_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_size, max_blocks_per_seq,
                                                 partition_tokens, ctypes.byref(n)), "pa_decode_workspace_bytes")
    return int(n.value)


def pa_set_decode_tuning(warps_per_cta: int = 0, stages: int = 0, ctas_per_sm: int = 0) -> None:
    _check(_lib_handle.pa_set_decode_tuning(warps_per_cta, stages, ctas_per_sm), "pa_set_decode_tuning")


def pa_get_device_status(stream=None) -> Tuple[int, int]:
    """Synchronise the stream; return (status, bits) and clear the device status word."""
    bits = ctypes.c_uint32(0)
    o = _opts(stream)
    st = _lib_handle.pa_get_device_status(ctypes.byref(o), ctypes.byref(bits))
    return int(st), int(bits.value)


def pa_debug_wait_selftest(timeout_ms: int, stream=None) -> None:
    o = _opts(stream, timeout_ms=timeout_ms)
    _check(_lib_handle.pa_debug_wait_selftest(ctypes.byref(o)), "pa_debug_wait_selftest")


# ---------------------------------------------------------------------------
# prepared calls: descriptors built once, for serving loops
# ---------------------------------------------------------------------------

class PreparedCall:
    """One library call whose descriptors (pa_tensor, pa_opts and scalars)
    are built once.  Calling it issues the same C call again, on ``stream``
    if given (else the stream it was prepared with), with no other Python
    work per call: for a serving loop that reuses the same buffers every
    step.  The tensors must stay alive and keep their storage, shapes and
    strides; their contents may change between calls.  Call it with the
    tensors' device current (as the preparing call had)."""

    def __init__(self, name: str, tensors, scalars, opts: PaOpts, keep):
        self._name = name
        self._fn = getattr(_lib_handle, name)
        self._structs = [_tensor(t) for t in tensors]
        self._opts = opts
        self._args = [ctypes.byref(t) for t in self._structs] + list(scalars) + [ctypes.byref(opts)]
        self._keep = keep  # the tensors, so their storage outlives this object

    def __call__(self, stream=None) -> None:
        if stream is not None:
            self._opts.stream = _stream_ptr(stream)
        _check(self._fn(*self._args), self._name)


def prepare_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> PreparedCall:
    """pa_reshape_and_cache, prepared (see PreparedCall)."""
    args = (key, value, k_cache, v_cache, slot_mapping)
    _device_index(args)
    return PreparedCall("pa_reshape_and_cache", args, [], _opts(stream), args)


def prepare_decode(out, query, k_cache, v_cache, block_tables, context_lens, scale: float, num_kv_heads: int,
                   workspace=None, partition_tokens: int = 0, stream=None, timeout_ms: int = 0) -> PreparedCall:
    """pa_decode, prepared (see PreparedCall)."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens)
    _device_index(args + (workspace,))
    return PreparedCall("pa_decode", args, [ctypes.c_float(scale), ctypes.c_int32(int(num_kv_heads))],
                        _opts(stream, workspace, partition_tokens, timeout_ms), args + (workspace,))


def prepare_reshape_and_cache_fp8(key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                                  stream=None) -> PreparedCall:
    """pa_reshape_and_cache_fp8, prepared (see PreparedCall)."""
    args = (key, value, k_cache, v_cache, slot_mapping, k_scale, v_scale)
    _device_index(args)
    return PreparedCall("pa_reshape_and_cache_fp8", args, [], _opts(stream), args)


def prepare_decode_fp8(out, query, k_cache, v_cache, block_tables, context_lens, scale: float, num_kv_heads: int,
                       k_scale, v_scale, workspace=None, partition_tokens: int = 0, stream=None,
                       timeout_ms: int = 0) -> PreparedCall:
    """pa_decode_fp8, prepared (see PreparedCall)."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens)
    _device_index(args + (k_scale, v_scale, workspace))
    call = PreparedCall("pa_decode_fp8", args, [ctypes.c_float(scale), ctypes.c_int32(int(num_kv_heads))],
                        _opts(stream, workspace, partition_tokens, timeout_ms), args + (k_scale, v_scale, workspace))
    # the two scale descriptors go between num_kv_heads and opts
    call._scales = [_tensor(k_scale), _tensor(v_scale)]
    call._args = call._args[:-1] + [ctypes.byref(t) for t in call._scales] + call._args[-1:]
    return call


def prepare_decode_cascade(out, query, k_cache, v_cache, block_tables, context_lens, group_start, group_blocks,
                           max_group_size: int, scale: float, num_kv_heads: int, workspace,
                           partition_tokens: int = 0, stream=None, timeout_ms: int = 0) -> PreparedCall:
    """pa_decode_cascade, prepared (see PreparedCall)."""
    args = (out, query, k_cache, v_cache, block_tables, context_lens, group_start, group_blocks)
    _device_index(args + (workspace,))
    return PreparedCall("pa_decode_cascade", args,
                        [ctypes.c_int32(int(max_group_size)), ctypes.c_float(scale), ctypes.c_int32(int(num_kv_heads))],
                        _opts(stream, workspace, partition_tokens, timeout_ms), args + (workspace,))


# ---------------------------------------------------------------------------
# host allocator
# ---------------------------------------------------------------------------

def _i64p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class Allocator:
    """Host block allocator of libpa (pa_alloc_* / pa_seq_*)."""

    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None):
        h = ctypes.c_void_p()
        if free_order is not None:
            self._order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if self._order.shape != (num_blocks,):
                raise ValueError("free_order must list every block once")
            ptr = _i32p(self._order)
        else:
            ptr = None
        _check(_lib_handle.pa_alloc_create(num_blocks, block_size, ptr, ctypes.byref(h)), "pa_alloc_create")
        self._h = h
        self._destroy = _lib_handle.pa_alloc_destroy  # kept: module globals may be gone at exit
        self.num_blocks = num_blocks
        self.block_size = block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        destroy = getattr(self, "_destroy", None)
        if h is not None and h.value and destroy is not None:
            destroy(h)
            self._h = None

    def add(self, seq: int) -> None:
        _check(_lib_handle.pa_seq_add(self._h, seq), "pa_seq_add")

    def append(self, seq: int, n: int):
        """Returns (slots int64 [n], copy-on-write pairs as a list of (src, dst))."""
        slots = np.zeros(max(n, 1), np.int64)
        pair = np.zeros(2, np.int64)
        ncow = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_append(self._h, seq, n, _i64p(slots), _i64p(pair), ctypes.byref(ncow)),
               "pa_seq_append")
        return slots[:n], ([(int(pair[0]), int(pair[1]))] if ncow.value else [])

    def append_batch(self, seqs: Sequence[int], counts: Sequence[int]):
        """Returns (slots of all tokens back to back, pairs int64 [n_cow, 2])."""
        ids = np.ascontiguousarray(np.asarray(seqs, np.int64))
        cnt = np.ascontiguousarray(np.asarray(counts, np.int32))
        slots = np.zeros(max(1, int(cnt.sum())), np.int64)
        pairs = np.zeros((max(1, len(ids)), 2), np.int64)
        ncow = ctypes.c_int32(0)
        ndone = ctypes.c_int32(0)
        st = _lib_handle.pa_seq_append_batch(self._h, _i64p(ids), _i32p(cnt), len(ids), _i64p(slots),
                                             _i64p(pairs), ctypes.byref(ncow), ctypes.byref(ndone))
        _check(st, f"pa_seq_append_batch (served {ndone.value} of {len(ids)})")
        return slots[: int(cnt.sum())], pairs[: ncow.value]

    def fork(self, parent: int, child: int) -> None:
        _check(_lib_handle.pa_seq_fork(self._h, parent, child), "pa_seq_fork")

    def add_prefix(self, seq: int, tokens: Sequence[int]) -> int:
        """Prefix caching: add a sequence on the longest registered chain of
        its prompt's full blocks; returns the number of tokens reused."""
        ids = np.ascontiguousarray(np.asarray(tokens, np.int64))
        n = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_add_prefix(self._h, seq, _i64p(ids) if ids.size else None, int(ids.size),
                                             ctypes.byref(n)), "pa_seq_add_prefix")
        return int(n.value)

    def append_tokens(self, seq: int, tokens: Sequence[int]):
        """Append tokens with known ids (blocks register when full)."""
        ids = np.ascontiguousarray(np.asarray(tokens, np.int64))
        n = int(ids.size)
        slots = np.zeros(max(n, 1), np.int64)
        pair = np.zeros(2, np.int64)
        ncow = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_append_tokens(self._h, seq, _i64p(ids) if n else _i64p(slots), n, _i64p(slots),
                                                _i64p(pair), ctypes.byref(ncow)), "pa_seq_append_tokens")
        return slots[:n], ([(int(pair[0]), int(pair[1]))] if ncow.value else [])

    def set_host_pool(self, num_host_blocks: int, host_free_order: Optional[Sequence[int]] = None) -> None:
        self._host_order = (np.ascontiguousarray(np.asarray(host_free_order, np.int32))
                            if host_free_order is not None else None)
        _check(_lib_handle.pa_alloc_set_host_pool(self._h, num_host_blocks,
                                                  _i32p(self._host_order) if self._host_order is not None else None),
               "pa_alloc_set_host_pool")
        self.num_host_blocks = num_host_blocks

    def _swap(self, fn, seq, where):
        cap = self.length(seq) // self.block_size + 2
        out = np.zeros((cap, 2), np.int64)
        n = ctypes.c_int32(0)
        _check(fn(self._h, seq, _i64p(out), cap, ctypes.byref(n)), where)
        return out[: n.value]

    def swap_out(self, seq: int):
        """(device, host) block pairs int64 [n, 2]; the device blocks are released."""
        return self._swap(_lib_handle.pa_seq_swap_out, seq, "pa_seq_swap_out")

    def swap_in(self, seq: int):
        """(host, device) block pairs int64 [n, 2]."""
        return self._swap(_lib_handle.pa_seq_swap_in, seq, "pa_seq_swap_in")

    def num_host_free(self) -> int:
        return int(_lib_handle.pa_alloc_num_host_free(self._h))

    def host_table(self, seq: int):
        cap = self.length(seq) // self.block_size + 1
        out = np.zeros(cap, np.int32)
        n = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_host_table(self._h, seq, _i32p(out), cap, ctypes.byref(n)), "pa_seq_host_table")
        return out[: n.value].tolist()

    def evictable(self):
        out = np.zeros(max(1, self.num_blocks), np.int32)
        n = ctypes.c_int32(0)
        _check(_lib_handle.pa_alloc_evictable(self._h, _i32p(out), self.num_blocks, ctypes.byref(n)),
               "pa_alloc_evictable")
        return out[: n.value].tolist()

    def free(self, seq: int) -> None:
        _check(_lib_handle.pa_seq_free(self._h, seq), "pa_seq_free")

    def length(self, seq: int) -> int:
        n = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_len(self._h, seq, ctypes.byref(n)), "pa_seq_len")
        return int(n.value)

    def block_table(self, seq: int):
        cap = self.length(seq) // self.block_size + 1
        out = np.zeros(cap, np.int32)
        n = ctypes.c_int32(0)
        _check(_lib_handle.pa_seq_block_table(self._h, seq, _i32p(out), cap, ctypes.byref(n)), "pa_seq_block_table")
        return out[: n.value].tolist()

    def block_tables(self, seqs: Sequence[int], max_blocks: int):
        """(tables int32 [n, max_blocks] padded with -1, context lengths int32 [n])."""
        ids = np.ascontiguousarray(np.asarray(seqs, np.int64))
        out = np.zeros((len(ids), max(max_blocks, 1)), np.int32)
        lens = np.zeros(max(len(ids), 1), np.int32)
        _check(_lib_handle.pa_alloc_block_tables(self._h, _i64p(ids), len(ids), _i32p(out), max_blocks,
                                                 _i32p(lens)), "pa_alloc_block_tables")
        return out[:, :max_blocks], lens[: len(ids)]

    def prefix_groups(self, seqs: Sequence[int], max_group_size: int):
        """(group_start int32 [n_groups + 1], group_blocks int32 [n_groups]):
        runs of consecutive batch sequences that share leading blocks, for
        ``pa_decode_cascade`` (pa_alloc_prefix_groups)."""
        ids = np.ascontiguousarray(np.asarray(seqs, np.int64))
        n = len(ids)
        gs = np.zeros(n + 1, np.int32)
        gb = np.zeros(max(n, 1), np.int32)
        ng = ctypes.c_int32(0)
        _check(_lib_handle.pa_alloc_prefix_groups(self._h, _i64p(ids) if n else None, n, int(max_group_size),
                                                  _i32p(gs), _i32p(gb), ctypes.byref(ng)), "pa_alloc_prefix_groups")
        return gs[: ng.value + 1], gb[: ng.value]

    def num_free(self) -> int:
        return int(_lib_handle.pa_alloc_num_free(self._h))

    def refcount(self, block: int) -> int:
        return int(_lib_handle.pa_block_refcount(self._h, block))

    def stats(self) -> dict:
        s = PaAllocStats()
        _check(_lib_handle.pa_alloc_get_stats(self._h, ctypes.byref(s)), "pa_alloc_get_stats")
        return {f: getattr(s, f) for f, _ in PaAllocStats._fields_}
