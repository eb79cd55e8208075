"""Oracle of the shared-prefix decode (test infrastructure; see the package
header).

The pages state that reference counts and copy-on-write let the parallel
samples of one prompt share both the prompt's memory and its computation
(CSDN discovery note, item 2, on the vLLM launch blog's "PagedAttention"
section).  The result of a decode is still plain attention over each
sequence's own context (``attention.paged_decode``); what a shared-prefix
decode changes is how it is reached: the prompt's blocks, which the
samples' block tables hold at the same indices, are attended once for all
samples, each sample attends its own remaining tokens, and the two partial
results are merged by log-sum-exp.  Two things are modelled here:

* ``prefix_groups`` — the library's rule for cutting a batch into groups of
  consecutive sequences that share leading blocks.  The pages give no rule;
  this library's: a group starts at a sequence, with its full blocks as the
  shared count; the next sequence joins while the group has fewer than
  ``max_group_size`` members, its table begins with at least one of the
  same full blocks, and joining keeps at least half of the shared count
  (the common count then becomes the shared count).  A group of one shares
  nothing.
* ``cascade_decode_rows`` — attention computed the shared-prefix way: per
  member, the partial result over tokens [0, 16 * shared) and the partial
  over [16 * shared, ctx), merged with ``attention.lse_merge``.  It must
  equal the plain definition (pinned in ``tests/test_oracle_cascade.py``).
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

from .attention import gather_sequence, lse_merge, partition_partials, widen


def prefix_groups(tables: Sequence[Sequence[int]], lens: Sequence[int], max_group_size: int,
                  block_size: int) -> Tuple[List[int], List[int]]:
    """Group starts ([n_groups + 1], the last entry = len(tables)) and the
    shared full-block count of each group, by the rule in the header."""
    n = len(tables)
    starts: List[int] = []
    shared: List[int] = []
    k = 0
    while k < n:
        start = k
        lead = list(tables[k])
        common = int(lens[k]) // block_size
        k += 1
        while k < n and k - start < max_group_size:
            cand = list(tables[k])
            cap = min(common, int(lens[k]) // block_size)
            c = 0
            while c < cap and cand[c] == lead[c]:
                c += 1
            if c == 0 or 2 * c < common:
                break
            common = c
            k += 1
        starts.append(start)
        shared.append(common if k - start > 1 else 0)
    starts.append(n)
    return starts, shared


def cascade_decode_rows(query, cache, block_tables, context_lens, group_start, group_blocks, scale: float,
                        query_dtype: str = "") -> Dict[int, np.ndarray]:
    """Outputs [H, D] (fp64) of every batch row, each computed as the
    log-sum-exp merge of its group's shared-prefix partial and its own
    suffix partial (a part with no tokens carries no weight)."""
    bs = cache.block_size
    qd = query_dtype or ("bf16" if cache.dtype == "fp8" else cache.dtype)
    res: Dict[int, np.ndarray] = {}
    for v in range(len(group_start) - 1):
        p_tokens = int(group_blocks[v]) * bs
        for i in range(int(group_start[v]), int(group_start[v + 1])):
            ctx = int(context_lens[i])
            q = widen(query[i], qd)
            k, vv = gather_sequence(cache, block_tables[i], ctx)
            h = q.shape[0]
            parts_o, parts_l = [], []
            for a, e in ((0, min(p_tokens, ctx)), (min(p_tokens, ctx), ctx)):
                if e > a:
                    o, lse = partition_partials(q, k[a:e], vv[a:e], scale, e - a)
                    parts_o.append(o[0])
                    parts_l.append(lse[0])
            if not parts_o:
                res[i] = np.zeros((h, q.shape[1]))
                continue
            res[i] = lse_merge(np.stack(parts_o), np.stack(parts_l))
    return res
