"""A paged KV cache on one GPU: the host allocator plus the device pools,
driven through the library's entry points.

This is bookkeeping around libpa: the allocator decides slots and
copy-on-write pairs on the host; the pairs are copied with pa_copy_blocks
and the tokens written with pa_reshape_and_cache (in that order, on one
stream); decode reads through int32 block tables.  Device memory comes from
torch; every byte is moved by the library's kernels.
"""

from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import (Allocator, pa_copy_blocks, pa_decode, pa_decode_cascade, pa_decode_cascade_workspace_bytes,
               pa_decode_fp8, pa_decode_workspace_bytes, pa_reshape_and_cache, pa_reshape_and_cache_fp8,
               prepare_decode, prepare_decode_cascade, prepare_decode_fp8, prepare_reshape_and_cache,
               prepare_reshape_and_cache_fp8)

_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}


class PagedKVCacheGPU:
    """K/V pools [num_blocks, num_kv_heads, block_size, head_size] on one device."""

    def __init__(self, num_blocks: int, num_kv_heads: int, head_size: int, dtype: str = "bf16",
                 block_size: int = 16, free_order: Optional[Sequence[int]] = None, device="cuda",
                 k_scale=None, v_scale=None):
        """dtype "fp8" stores e4m3 codes and needs per-kv-head k_scale/v_scale
        (float32 [num_kv_heads])."""
        self.num_blocks, self.num_kv_heads, self.head_size = num_blocks, num_kv_heads, head_size
        self.block_size, self.dtype, self.device = block_size, dtype, torch.device(device)
        shape = (num_blocks, num_kv_heads, block_size, head_size)
        self.k_cache = torch.empty(shape, dtype=_DT[dtype], device=self.device)
        self.v_cache = torch.empty(shape, dtype=_DT[dtype], device=self.device)
        self.alloc = Allocator(num_blocks, block_size, free_order)
        self._ws = None
        self._cws = None
        self.k_scale = self.v_scale = None
        if dtype == "fp8":
            if k_scale is None or v_scale is None:
                raise ValueError("an fp8 cache needs k_scale and v_scale")
            self.k_scale = torch.as_tensor(k_scale, dtype=torch.float32).to(self.device).contiguous()
            self.v_scale = torch.as_tensor(v_scale, dtype=torch.float32).to(self.device).contiguous()

    # -- host bookkeeping ------------------------------------------------------
    def add(self, seq: int) -> None:
        self.alloc.add(seq)

    def fork(self, parent: int, child: int) -> None:
        self.alloc.fork(parent, child)

    def free(self, seq: int) -> None:
        self.alloc.free(seq)

    def append(self, seqs: Sequence[int], counts: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
        """Reserve slots for counts[k] new tokens of seqs[k]; returns (slots
        int64 [sum(counts)], copy-on-write pairs int64 [n, 2])."""
        return self.alloc.append_batch(seqs, counts)

    def block_tables(self, seqs: Sequence[int], max_blocks: int) -> Tuple[np.ndarray, np.ndarray]:
        return self.alloc.block_tables(seqs, max_blocks)

    # -- device steps -------------------------------------------------------------
    def write(self, slots: torch.Tensor, key: torch.Tensor, value: torch.Tensor,
              pairs: Optional[torch.Tensor] = None, stream=None) -> None:
        """Copy-on-write copies first (they must precede writes into the
        copied blocks), then the tokens' K/V at their slots."""
        if pairs is not None and pairs.shape[0]:
            pa_copy_blocks(self.k_cache, self.v_cache, pairs, stream=stream)
        if self.dtype == "fp8":
            pa_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slots, self.k_scale, self.v_scale,
                                     stream=stream)
        else:
            pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots, stream=stream)

    def workspace(self, num_seqs: int, num_heads: int, max_blocks: int, partition_tokens: int = 0):
        """Split scratch for ``decode``, grown on demand and reused by every
        call (zero-filled when allocated: its merge counters must start at
        zero, and every call leaves them zero): decodes that may overlap on
        the GPU (different streams) must each pass a workspace of their own."""
        n = pa_decode_workspace_bytes(num_seqs, num_heads, self.num_kv_heads, self.head_size, max_blocks,
                                      partition_tokens)
        if n == 0:
            return None
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        return self._ws

    def prefix_groups(self, seqs: Sequence[int], num_heads: int):
        """Groups of consecutive batch sequences that share leading blocks
        (forks of one prompt), for ``decode_shared``: returns
        (group_start, group_blocks) as int32 numpy arrays and the group width
        to pass as max_group_size (the widest group found, rounded up to a
        power of two, at most 8 query rows per kv head in all)."""
        g = num_heads // self.num_kv_heads
        widest = max(1, 8 // g)
        gs, gb = self.alloc.prefix_groups(seqs, widest)
        sizes = gs[1:] - gs[:-1]
        need = int(sizes[gb > 0].max()) if (gb > 0).any() else 1
        m = 1
        while m < need:
            m *= 2
        if m != widest:
            gs, gb = self.alloc.prefix_groups(seqs, m)
        return gs, gb, m

    def shared_workspace(self, num_seqs: int, num_heads: int, max_group_size: int, partition_tokens: int = 0):
        """Zero-filled workspace for ``decode_shared`` (grown on demand,
        reused by every call on one stream)."""
        n = pa_decode_cascade_workspace_bytes(num_seqs, num_heads, self.num_kv_heads, self.head_size, max_group_size,
                                              partition_tokens)
        if self._cws is None or self._cws.numel() < n:
            self._cws = torch.zeros(n, dtype=torch.uint8, device=self.device)
        return self._cws

    def decode_shared(self, out: torch.Tensor, query: torch.Tensor, block_tables: torch.Tensor,
                      context_lens: torch.Tensor, group_start: torch.Tensor, group_blocks: torch.Tensor,
                      max_group_size: int, scale: float, partition_tokens: int = 0, stream=None,
                      workspace=None) -> torch.Tensor:
        """Decode with each group's shared prompt blocks read once for all
        of its samples (pa_decode_cascade)."""
        if workspace is None:
            workspace = self.shared_workspace(query.shape[0], query.shape[1], max_group_size, partition_tokens)
        pa_decode_cascade(out, query, self.k_cache, self.v_cache, block_tables, context_lens, group_start,
                          group_blocks, max_group_size, scale, self.num_kv_heads, workspace,
                          partition_tokens=partition_tokens, stream=stream)
        return out

    def decode(self, out: torch.Tensor, query: torch.Tensor, block_tables: torch.Tensor,
               context_lens: torch.Tensor, scale: float, partition_tokens: int = 0, stream=None,
               workspace=None) -> torch.Tensor:
        if workspace is None:
            workspace = self.workspace(query.shape[0], query.shape[1], block_tables.shape[1], partition_tokens)
        if self.dtype == "fp8":
            pa_decode_fp8(out, query, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                          self.num_kv_heads, self.k_scale, self.v_scale, workspace=workspace,
                          partition_tokens=partition_tokens, stream=stream)
        else:
            pa_decode(out, query, self.k_cache, self.v_cache, block_tables, context_lens, scale, self.num_kv_heads,
                      workspace=workspace, partition_tokens=partition_tokens, stream=stream)
        return out

    def prepare_step(self, slots: torch.Tensor, key: torch.Tensor, value: torch.Tensor, out: torch.Tensor,
                     query: torch.Tensor, block_tables: torch.Tensor, context_lens: torch.Tensor, scale: float,
                     partition_tokens: int = 0, stream=None, workspace=None, groups=None):
        """One serving step (the new tokens' cache write, then the decode)
        over fixed buffers, as prepared calls (descriptors built once): the
        returned function runs the step again on the buffers' current
        contents.  ``groups``: (group_start, group_blocks, max_group_size)
        device tensors and width for a shared-prefix decode."""
        if self.dtype == "fp8":
            write = prepare_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slots, self.k_scale,
                                                  self.v_scale, stream=stream)
        else:
            write = prepare_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots, stream=stream)
        if groups is not None:
            gs, gb, mg = groups
            if workspace is None:
                workspace = self.shared_workspace(query.shape[0], query.shape[1], mg, partition_tokens)
            dec = prepare_decode_cascade(out, query, self.k_cache, self.v_cache, block_tables, context_lens, gs, gb,
                                         mg, scale, self.num_kv_heads, workspace, partition_tokens, stream=stream)
        else:
            if workspace is None:
                workspace = self.workspace(query.shape[0], query.shape[1], block_tables.shape[1], partition_tokens)
            if self.dtype == "fp8":
                dec = prepare_decode_fp8(out, query, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                                         self.num_kv_heads, self.k_scale, self.v_scale, workspace, partition_tokens,
                                         stream=stream)
            else:
                dec = prepare_decode(out, query, self.k_cache, self.v_cache, block_tables, context_lens, scale,
                                     self.num_kv_heads, workspace, partition_tokens, stream=stream)
        return PreparedStep(write if slots.numel() > 0 else None, dec)


class PreparedStep:
    """A serving step as prepared library calls: ``write`` (the new tokens'
    cache write, None when the step appends nothing) and ``decode``; calling
    the step runs both, in that order, on the stream they were prepared
    with."""

    def __init__(self, write, decode):
        self.write = write
        self.decode = decode

    def __call__(self) -> None:
        if self.write is not None:
            self.write()
        self.decode()
