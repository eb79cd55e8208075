"""Replay a seeded workload through the oracle block manager and cache
(test infrastructure; see the package header).

Each request of a ``workloads.Plan`` is applied in order: ``add`` and
``fork`` go to the block manager; ``append`` asks it for slots, performs the
copy-on-write copies it reports (before the write, since the write lands in
the copied block), then writes the tokens' K/V at those slots.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

from workloads import AddOp, ForkOp, AppendOp, Plan, kv_scales, stream_kv

from .allocator import BlockAllocator
from .attention import widen
from .cache import PagedKVCache
from .quant import quantize_kv


@dataclass
class ReplayLog:
    """Per append request, in order: (seq, slots, copy-on-write pairs)."""

    appends: List[Tuple[int, List[int], List[Tuple[int, int]]]] = field(default_factory=list)


def replay(plan: Plan, stop_after: Optional[int] = None, include_step: bool = True,
           write_values: bool = True):
    """Returns (allocator, cache, log).  ``stop_after`` counts requests of
    setup+step in order; ``write_values=False`` skips the K/V bytes (for
    allocator-only checks of large workloads)."""
    w = plan.workload
    alloc = BlockAllocator(plan.num_blocks, w.block_size, plan.free_order)
    if w.cache_dtype == "fp8":
        ks, vs = kv_scales(plan)
        cache = PagedKVCache(plan.num_blocks, w.num_kv_heads, w.head_size, w.block_size, "fp8", ks, vs)
    else:
        cache = PagedKVCache(plan.num_blocks, w.num_kv_heads, w.head_size, w.block_size, w.dtype)
    log = ReplayLog()
    ops = list(plan.setup_ops) + (list(plan.step_ops) if include_step else [])
    if stop_after is not None:
        ops = ops[:stop_after]
    for op in ops:
        if isinstance(op, AddOp):
            alloc.add(op.seq)
        elif isinstance(op, ForkOp):
            alloc.fork(op.parent, op.child)
        elif isinstance(op, AppendOp):
            slots, cow = alloc.append(op.seq, op.n)
            log.appends.append((op.seq, slots, cow))
            if write_values:
                cache.copy_blocks(cow)
                k, v = stream_kv(plan, op.stream, op.start, op.n)
                if w.cache_dtype == "fp8":  # the write quantizes the bf16 inputs
                    k = quantize_kv(widen(k, w.dtype).astype(np.float32), cache.k_scale)
                    v = quantize_kv(widen(v, w.dtype).astype(np.float32), cache.v_scale)
                cache.write(slots, k, v)
        else:
            raise TypeError(op)
    return alloc, cache, log


def block_table_array(alloc: BlockAllocator, seqs, max_blocks: int) -> np.ndarray:
    """int32 [len(seqs), max_blocks]; entries past a table's end are -1."""
    out = np.full((len(seqs), max_blocks), -1, np.int32)
    for r, s in enumerate(seqs):
        t = alloc.block_table(int(s))
        out[r, :len(t)] = t
    return out
