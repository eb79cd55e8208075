"""CPU oracle for paged KV cache attention — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct NumPy code (fp64 for all floating point) that
states what the PagedAttention hot path computes, written from the pages'
definitions:

* ``allocator``  — the block manager: fixed-size KV blocks, a per-sequence
  block table from logical to physical blocks, blocks handed out on demand,
  reference counts and copy-on-write for shared prompt blocks
  (vLLM launch blog, "PagedAttention" section, as summarised on the CSDN
  discovery note, item 2; agientry.com overview, opening section).
* ``cache``      — physical K/V storage and the two byte-moving steps: the
  per-token cache write by slot and the whole-block copy of copy-on-write.
* ``quant``      — FP8 (e4m3) codes of a quantized KV cache with per-head
  scales (the pages only say the KV cache can be quantized; gitcode repo
  walkthrough, section 三 "量化").
* ``attention``  — single-query attention softmax(q K^T * scale) V over the
  tokens a block table names, walked logically, in fp64; and the
  log-sum-exp merge of per-partition partial results.
* ``prefill``    — multi-token (chunked-prefill) attention: every new token
  of a sequence attends causally over its cache (gitcode repo walkthrough,
  section 2.2), in fp64.
* ``replay``     — applies a seeded workload's requests to the allocator and
  cache models.
* the allocator also models prefix caching (hash-free keys: parent block and
  token ids) and swapping to a host block pool.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  It shares no
code with the CUDA path and imports nothing from it.  Inputs come from the
seeded generators in ``workloads`` (which hold none of the method's
arithmetic) or from the tests themselves.

Parity status: every function here is pinned by tests in ``tests/test_oracle_*``
against closed forms, invariants, brute force or an independent library
routine; none is "parity unpinned".
"""

from .allocator import BlockAllocator, OutOfBlocks, AllocatorError  # noqa: F401
from .cache import PagedKVCache  # noqa: F401
from .quant import e4m3_decode, e4m3_encode, quantize_kv  # noqa: F401
from .attention import (  # noqa: F401
    widen,
    paged_decode,
    paged_decode_rows,
    gather_sequence,
    attend_contiguous,
    partition_partials,
    lse_merge,
)
from .prefill import paged_prefill, paged_prefill_seqs  # noqa: F401
