"""Prefix caching end to end on the GPU.

Requests that share a system prompt reuse its cached full blocks (C++
allocator: pa_seq_add_prefix / pa_seq_append_tokens) and write only the K/V
of the tokens the cache does not hold; some requests are freed and new ones
arrive, so evictable blocks are reused by later hits and evicted blocks are
overwritten.  The block tables must equal the oracle allocator's, and every
request's decode must match the oracle's attention over its logical history
(max-abs <= 1e-2, bf16).  A token's K/V depends on its whole prefix, so the
values of a system-prompt position come from that prompt's stream and those
of a request's own tokens from the request's stream.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import check_status_clean, to_device_values, to_host_raw
from oracle.allocator import BlockAllocator
from oracle.attention import paged_decode, widen
from oracle.cache import PagedKVCache
from oracle.replay import block_table_array
from workloads import to_bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
HK, H, D, BS, NB = 8, 8, 128, 16, 700


def _values(stream, start, n):
    """K and V (bf16 bits) of positions [start, start+n) of a token stream."""
    ks, vs = [], []
    for p in range(start, start + n):
        r = np.random.default_rng([999, stream, p])
        ks.append(r.standard_normal((HK, D), dtype=np.float32))
        vs.append(r.standard_normal((HK, D), dtype=np.float32))
    if not n:
        return np.zeros((0, HK, D), np.uint16), np.zeros((0, HK, D), np.uint16)
    return to_bf16_bits(np.stack(ks)), to_bf16_bits(np.stack(vs))


def test_prefix_cache_reuse_and_eviction():
    rng = np.random.default_rng(11)
    sys_len = [300, 517, 64]
    order = rng.permutation(NB).astype(np.int32)
    c = pa.Allocator(NB, BS, order)
    o = BlockAllocator(NB, BS, order)
    cache_o = PagedKVCache(NB, HK, D, BS, "bf16")
    kc = torch.empty(NB, HK, BS, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.empty_like(kc)
    prompts = {}
    live = []
    total_hit = 0

    def request(r, sysk, own):
        nonlocal total_hit
        toks = [1000 * (sysk + 1) + t for t in range(sys_len[sysk])] + [10 ** 6 * (r + 1) + t for t in range(own)]
        hit = c.add_prefix(r, toks)
        assert o.add_prefix(r, toks) == hit
        total_hit += hit
        slots, cow = c.append_tokens(r, toks[hit:])
        so, co = o.append_tokens(r, toks[hit:])
        assert slots.tolist() == so and cow == co == []
        # K/V of the positions the cache does not hold
        n_sys = max(0, sys_len[sysk] - hit)
        k1, v1 = _values(100 + sysk, hit, n_sys)
        k2, v2 = _values(200 + r, max(0, hit - sys_len[sysk]), len(toks) - hit - n_sys)
        k, v = np.concatenate([k1, k2]), np.concatenate([v1, v2])
        cache_o.write(so, k, v)
        pa.pa_reshape_and_cache(to_device_values(k, "bf16", DEV), to_device_values(v, "bf16", DEV), kc, vc,
                                torch.from_numpy(slots).to(DEV))
        prompts[r] = toks
        live.append(r)

    for r in range(12):
        request(r, r % 3, int(rng.integers(1, 40)))
    for r in (1, 4, 7, 2):  # free some: their private blocks go free, shared ones stay or become evictable
        c.free(r)
        o.free(r)
        live.remove(r)
    for r in range(12, 30):  # more requests: hits on held and evictable blocks, then eviction under pressure
        request(r, int(rng.integers(0, 3)), int(rng.integers(1, 200)))
    assert total_hit > 0
    assert c.stats()["num_cached"] == o.num_cached() and c.evictable() == list(o._evictable)

    seqs = sorted(live)
    max_nb = max(len(prompts[s]) for s in seqs) // BS + 1
    tables, lens = c.block_tables(seqs, max_nb)
    assert np.array_equal(tables, block_table_array(o, seqs, max_nb))
    q = to_bf16_bits(rng.standard_normal((len(seqs), H, D)).astype(np.float32))
    out = torch.empty(len(seqs), H, D, dtype=torch.bfloat16, device=DEV)
    n = pa.pa_decode_workspace_bytes(len(seqs), H, HK, D, max_nb, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    pa.pa_decode(out, to_device_values(q, "bf16", DEV), kc, vc, torch.from_numpy(tables).to(DEV),
                 torch.from_numpy(lens).to(DEV), 1 / math.sqrt(D), HK, workspace=ws)
    check_status_clean()
    ref = paged_decode(q, cache_o, tables, lens, 1 / math.sqrt(D))
    got = widen(to_host_raw(out, "bf16"), "bf16")
    assert float(np.max(np.abs(got - ref))) <= 1e-2
