"""Oracle physical KV storage (test infrastructure; see the package header).

A block holds the K (and, separately, the V) of ``block_size`` consecutive
tokens for every KV head: the pages state that one block stores BLOCK_SIZE
tokens of one head, e.g. 2048 elements per block per head at block size 16
and head size 128 (gitcode repo walkthrough, section 2.1 "PagedAttention").
Values are kept as their raw storage bits (float32, bfloat16 bit patterns in
uint16, or FP8 e4m3 codes in uint8 with per-kv-head scales) so that
byte-moving steps can be compared bit for bit.

* ``write``: the cache write — token t's K/V for head h go to slot
  ``slots[t]``, i.e. block ``slot // bs``, offset ``slot % bs``; slot -1 means
  "no write" (a padding token).
* ``copy_blocks``: the copy of copy-on-write — the whole block (all heads, all
  offsets, K and V) of ``src`` is copied to ``dst``.

Only blocks that were written are held, so a 40 GB pool costs only what the
sequences use.  Offsets never written are tracked, and reading them is an
error: nothing in the method reads a slot before it is written.
"""

from __future__ import annotations

from typing import Dict, Iterable, Sequence, Tuple

import numpy as np


class PagedKVCache:
    def __init__(self, num_blocks: int, num_kv_heads: int, head_size: int, block_size: int, dtype: str,
                 k_scale=None, v_scale=None):
        if dtype not in ("f32", "bf16", "fp8"):
            raise ValueError("dtype must be 'f32', 'bf16' or 'fp8'")
        if dtype == "fp8" and (k_scale is None or v_scale is None):
            raise ValueError("an fp8 cache needs per-head k_scale and v_scale")
        self.num_blocks = num_blocks
        self.num_kv_heads = num_kv_heads
        self.head_size = head_size
        self.block_size = block_size
        self.dtype = dtype
        self.raw_dtype = {"f32": np.float32, "bf16": np.uint16, "fp8": np.uint8}[dtype]
        # fp8: stored codes are value / scale[h] (see oracle.quant)
        self.k_scale = None if k_scale is None else np.asarray(k_scale, np.float32)
        self.v_scale = None if v_scale is None else np.asarray(v_scale, np.float32)
        self._k: Dict[int, np.ndarray] = {}
        self._v: Dict[int, np.ndarray] = {}
        self._written: Dict[int, np.ndarray] = {}

    def _page(self, block: int):
        if not 0 <= block < self.num_blocks:
            raise IndexError(f"block {block} outside the pool of {self.num_blocks}")
        if block not in self._k:
            shape = (self.num_kv_heads, self.block_size, self.head_size)
            self._k[block] = np.zeros(shape, self.raw_dtype)
            self._v[block] = np.zeros(shape, self.raw_dtype)
            self._written[block] = np.zeros(self.block_size, bool)
        return self._k[block], self._v[block], self._written[block]

    def write(self, slots: Sequence[int], key: np.ndarray, value: np.ndarray) -> None:
        """key/value: [T, H_kv, D] raw storage; slots: [T] int."""
        slots = np.asarray(slots, dtype=np.int64)
        key = np.asarray(key)
        value = np.asarray(value)
        if key.shape != value.shape or key.shape[0] != slots.shape[0]:
            raise ValueError("key, value and slots disagree in length")
        if key.shape[1:] != (self.num_kv_heads, self.head_size) or key.dtype != self.raw_dtype:
            raise ValueError("key/value shape or storage type does not match the cache")
        bs = self.block_size
        for t, s in enumerate(slots.tolist()):
            if s == -1:
                continue
            if s < 0:
                raise IndexError(f"slot {s} is negative")
            kb, vb, wr = self._page(s // bs)
            kb[:, s % bs, :] = key[t]
            vb[:, s % bs, :] = value[t]
            wr[s % bs] = True

    def copy_blocks(self, pairs: Iterable[Tuple[int, int]]) -> None:
        for src, dst in pairs:
            ks, vs, ws = self._page(int(src))
            kd, vd, wd = self._page(int(dst))
            kd[...] = ks
            vd[...] = vs
            wd[...] = ws

    def copy_blocks_to(self, dst: "PagedKVCache", pairs: Iterable[Tuple[int, int]]) -> None:
        """Whole-block copies into another pool (swap out / swap in): for each
        (src, dst) pair, dst's block becomes a copy of this cache's block."""
        for s_, d_ in pairs:
            ks, vs, ws = self._page(int(s_))
            kd, vd, wd = dst._page(int(d_))
            kd[...] = ks
            vd[...] = vs
            wd[...] = ws

    def blocks(self):
        return sorted(self._k.keys())

    def k_page(self, block: int) -> np.ndarray:
        """Raw K of a block, [H_kv, bs, D]."""
        return self._page(block)[0]

    def v_page(self, block: int) -> np.ndarray:
        return self._page(block)[1]

    def written(self, block: int) -> np.ndarray:
        return self._page(block)[2]

    def read_token(self, slot: int) -> Tuple[np.ndarray, np.ndarray]:
        """Raw K and V of one slot, each [H_kv, D]."""
        bs = self.block_size
        kb, vb, wr = self._page(slot // bs)
        if not wr[slot % bs]:
            raise IndexError(f"slot {slot} was never written")
        return kb[:, slot % bs, :], vb[:, slot % bs, :]
