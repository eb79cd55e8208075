"""Oracle multi-token (chunked-prefill) attention over a paged KV cache
(test infrastructure; see the package header).

The pages name chunked prefill as one of the serving-loop optimisations: a
long prompt's prefill is cut into chunks that run in the same step as decode
requests, so that one long prompt does not take a whole step (gitcode repo
walkthrough, section 2.2 "连续批处理、Chunked Prefill 与 Prefix Caching").
The attention of such a step is still the definition the pages give for the
kernel (section 2.1: query-key dot product, softmax, weighted sum of V over
K/V gathered through the block table), applied to every new token with the
causal rule that a token sees itself and the tokens before it.  Reading taken
(the pages give no formula for the chunked step):

    sequence i brings n_i = query_start[i+1] - query_start[i] new tokens, at
    logical positions c_i + j (j = 0 .. n_i - 1, c_i = ctx_i - n_i); their
    K/V are already in the cache (the step's cache write runs first);
    query row r = query_start[i] + j, head h, kv head g = h // G:
        s_t = scale * <q[r,h], K_i[t, g]>        t = 0 .. c_i + j
        out[r,h] = sum_t softmax(s)_t V_i[t, g]

A decode request is n_i = 1 (the row is exactly the decode definition); a
whole prompt is c_i = 0 (plain causal self-attention); n_i = 0 contributes no
rows.  Everything is fp64 over exactly widened stored values.
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np

from .attention import gather_sequence, widen


def _rows_of_sequence(q: np.ndarray, k: np.ndarray, v: np.ndarray, prior: int, scale: float) -> np.ndarray:
    """q [n, H, D] (fp64) of the new tokens at positions prior .. prior+n-1;
    k/v [ctx, H_kv, D] with ctx = prior + n.  Returns [n, H, D] fp64."""
    n, h_q, d = q.shape
    ctx, h_kv, _ = k.shape
    if h_q % h_kv:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    group = h_q // h_kv
    out = np.zeros((n, h_q, d), np.float64)
    if n == 0:
        return out
    pos = prior + np.arange(n)  # logical position of each query row
    allowed = np.arange(ctx)[None, :] <= pos[:, None]  # [n, ctx] causal rule
    for h in range(h_q):
        g = h // group
        s = scale * (q[:, h, :] @ k[:, g, :].T)  # [n, ctx]
        s = np.where(allowed, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, g, :]
    return out


def paged_prefill_seqs(query, cache, block_tables, context_lens, query_start, scale: float,
                       seqs: Iterable[int], query_dtype: str = "") -> Dict[int, np.ndarray]:
    """Outputs [n_i, H, D] (fp64) of the chosen sequences.  ``query`` is
    [num_rows, H, D] in the cache's storage type (bf16 for an fp8 cache,
    unless given); ``query_start`` int [B + 1]."""
    qd = query_dtype or ("bf16" if cache.dtype == "fp8" else cache.dtype)
    res: Dict[int, np.ndarray] = {}
    for i in seqs:
        i = int(i)
        a, e = int(query_start[i]), int(query_start[i + 1])
        ctx = int(context_lens[i])
        n = e - a
        if n < 0 or n > ctx:
            raise ValueError(f"sequence {i}: {n} new tokens with context {ctx}")
        k, v = gather_sequence(cache, block_tables[i], ctx)
        res[i] = _rows_of_sequence(widen(query[a:e], qd), k, v, ctx - n, scale)
    return res


def paged_prefill(query, cache, block_tables, context_lens, query_start, scale: float,
                  query_dtype: Optional[str] = "") -> np.ndarray:
    """All rows: out [num_rows, H, D] fp64, row r of sequence i at
    ``query_start[i] + j``."""
    b = len(context_lens)
    out = np.zeros(tuple(query.shape), np.float64)
    rows = paged_prefill_seqs(query, cache, block_tables, context_lens, query_start, scale, range(b),
                              query_dtype or "")
    for i in range(b):
        out[int(query_start[i]):int(query_start[i + 1])] = rows[i]
    return out
