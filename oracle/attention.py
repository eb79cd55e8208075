"""Oracle single-query (decode) attention over a paged KV cache
(test infrastructure; see the package header).

PagedAttention changes where K and V are stored, not what attention computes:
the pages describe the kernel as the ordinary three steps — the query-key dot
product, the softmax normalisation and the weighted sum of values — carried
out over K/V that the block table gathers from non-contiguous blocks
(gitcode repo walkthrough, section 2.1 "PagedAttention"; vLLM launch blog,
"PagedAttention" section, on the CSDN discovery note, item 2).  So the oracle
is that definition written out in fp64:

    for sequence i and query head h, with kv head g = h // G (G = H / H_kv):
        s_t = scale * <q[i,h], K_i[t, g]>            t = 0 .. ctx_i - 1
        p   = exp(s - max s) / sum exp(s - max s)
        out[i,h] = sum_t p_t V_i[t, g]

where K_i[t] is read from block ``block_table[i][t // bs]`` at offset
``t % bs``.  Readings of points the pages leave open:

* GQA: query heads map to KV heads in contiguous groups, ``g = h // G``.
* ``context_lens`` counts every token attended, including the one written
  in this step; a sequence with ``ctx = 0`` yields an all-zero output row.
* no mask, bias, soft-cap or window: plain full attention over ctx tokens.
* q, K and V are widened exactly from their storage type to fp64.

``partition_partials`` and ``lse_merge`` restate the split-context algebra
used for long contexts (per partition p: m_p, l_p = sum exp(s - m_p),
o_p = sum exp(s - m_p) v / l_p, lse_p = m_p + ln l_p; merged
out = sum_p exp(lse_p - LSE) o_p with LSE = log sum_p exp(lse_p)); the pages
do not describe this step, so it is pinned only by its agreement with the
unsplit definition.
"""

from __future__ import annotations

from typing import Dict, Iterable, List, Sequence, Tuple

import numpy as np


def widen(raw: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values (float32, bf16 bits, or e4m3 codes
    without their scale) to fp64."""
    raw = np.asarray(raw)
    if dtype == "f32":
        return raw.astype(np.float64)
    if dtype == "fp8":
        from .quant import e4m3_decode

        return e4m3_decode(raw)
    if dtype == "bf16":
        bits = raw.astype(np.uint16).astype(np.uint32) << np.uint32(16)
        return bits.view(np.float32).astype(np.float64)
    raise ValueError(dtype)


def gather_sequence(cache, block_table: Sequence[int], ctx: int) -> Tuple[np.ndarray, np.ndarray]:
    """Walk a block table logically: token t is at block ``table[t // bs]``,
    offset ``t % bs``.  Returns fp64 K and V, each [ctx, H_kv, D]."""
    bs = cache.block_size
    hk, d = cache.num_kv_heads, cache.head_size
    k = np.empty((ctx, hk, d), np.float64)
    v = np.empty((ctx, hk, d), np.float64)
    for t0 in range(0, ctx, bs):
        b = int(block_table[t0 // bs])
        n = min(bs, ctx - t0)
        if not cache.written(b)[:n].all():
            raise IndexError(f"block {b} read at offsets that were never written")
        k[t0:t0 + n] = widen(cache.k_page(b)[:, :n, :], cache.dtype).transpose(1, 0, 2)
        v[t0:t0 + n] = widen(cache.v_page(b)[:, :n, :], cache.dtype).transpose(1, 0, 2)
    if cache.dtype == "fp8":  # dequantize: code value times the head's scale
        k *= cache.k_scale.astype(np.float64)[None, :, None]
        v *= cache.v_scale.astype(np.float64)[None, :, None]
    return k, v


def attend_contiguous(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """q [H, D], k/v [ctx, H_kv, D] (fp64) -> out [H, D] fp64."""
    h_q, d = q.shape
    ctx, h_kv, _ = k.shape
    if h_q % h_kv:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    group = h_q // h_kv
    out = np.zeros((h_q, d), np.float64)
    if ctx == 0:
        return out
    for h in range(h_q):
        g = h // group
        s = scale * (k[:, g, :] @ q[h])
        p = np.exp(s - s.max())
        p /= p.sum()
        out[h] = p @ v[:, g, :]
    return out


def paged_decode_rows(query, cache, block_tables, context_lens, scale: float,
                      seqs: Iterable[int], query_dtype: str = "") -> Dict[int, np.ndarray]:
    """Outputs [H, D] (fp64) of the chosen batch rows only.  The query is in
    the cache's storage type, or bf16 for an fp8 cache (unless given)."""
    qd = query_dtype or ("bf16" if cache.dtype == "fp8" else cache.dtype)
    res: Dict[int, np.ndarray] = {}
    for i in seqs:
        i = int(i)
        ctx = int(context_lens[i])
        q = widen(query[i], qd)
        k, v = gather_sequence(cache, block_tables[i], ctx)
        res[i] = attend_contiguous(q, k, v, scale)
    return res


def paged_decode(query, cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """query [B, H, D] raw storage; block_tables [B][>= nb_i] ints;
    context_lens [B].  Returns out [B, H, D] fp64."""
    b = len(context_lens)
    rows = paged_decode_rows(query, cache, block_tables, context_lens, scale, range(b))
    return np.stack([rows[i] for i in range(b)]) if b else np.zeros((0,) + tuple(query.shape[1:]))


def partition_partials(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                       partition_tokens: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-partition partial results of one sequence: partitions are
    [p*P, (p+1)*P) intersected with [0, ctx).  Returns (o [P, H, D], lse [P, H])."""
    h_q, d = q.shape
    ctx, h_kv, _ = k.shape
    group = h_q // h_kv
    n_part = -(-ctx // partition_tokens)
    o = np.zeros((n_part, h_q, d))
    lse = np.zeros((n_part, h_q))
    for p in range(n_part):
        a, e = p * partition_tokens, min(ctx, (p + 1) * partition_tokens)
        for h in range(h_q):
            g = h // group
            s = scale * (k[a:e, g, :] @ q[h])
            m = s.max()
            w = np.exp(s - m)
            l_sum = w.sum()
            o[p, h] = (w @ v[a:e, g, :]) / l_sum
            lse[p, h] = m + np.log(l_sum)
    return o, lse


def lse_merge(o: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """Merge partials: o [P, H, D], lse [P, H] -> [H, D].  Partitions with
    lse = -inf (no tokens) carry no weight."""
    m = np.max(lse, axis=0)
    total = m + np.log(np.sum(np.exp(lse - m), axis=0))
    w = np.exp(lse - total)  # [P, H]
    return np.einsum("ph,phd->hd", w, o)
