"""Pins for the oracle decode attention and its split-context merge.

The pages print no numeric example of attention, so the oracle is pinned by
(gitcode repo walkthrough, section 2.1: PagedAttention is the usual QK dot
product, softmax and weighted sum of V over K/V gathered from blocks):
  * agreement with torch's scaled_dot_product_attention (fp64, contiguous
    K/V, enable_gqa) — an independent library formulation, which also fixes
    the grouped-query head map h -> h // G;
  * bit-identical output under any permutation of physical blocks;
  * closed forms: identical keys -> mean of V; ctx = 1 -> v; q = 0 -> mean of
    V; constant V -> that constant; one dominant logit -> its v;
  * scalar brute force with the math module on tiny inputs;
  * the split-context merge equals the unsplit result.
Planted mistakes (wrong head map, missing scale, a dropped token, wrong block
offset) are run against these pins to show that each is caught.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle.cache import PagedKVCache
from workloads import to_bf16_bits


def _paged_setup(rng, ctxs, h, hk, d, bs=16, dtype="f32", spare=3):
    """Random contiguous K/V per sequence, scattered into a pool through a
    random permutation of physical blocks.  Returns (cache, tables, q_raw,
    k_list, v_list) where k_list/v_list are the fp64 contiguous values."""
    nbs = [-(-c // bs) for c in ctxs]
    nb = sum(nbs) + spare
    perm = rng.permutation(nb)
    cache = PagedKVCache(nb, hk, d, bs, dtype)
    tables, ks, vs = [], [], []
    off = 0
    for c, n in zip(ctxs, nbs):
        table = [int(x) for x in perm[off:off + n]]
        off += n
        tables.append(table)
        k = rng.standard_normal((c, hk, d)).astype(np.float32)
        v = rng.standard_normal((c, hk, d)).astype(np.float32)
        if dtype == "bf16":
            k, v = to_bf16_bits(k), to_bf16_bits(v)
        slots = [table[t // bs] * bs + t % bs for t in range(c)]
        cache.write(slots, k, v)
        ks.append(att.widen(k, dtype))
        vs.append(att.widen(v, dtype))
    q = rng.standard_normal((len(ctxs), h, d)).astype(np.float32)
    if dtype == "bf16":
        q = to_bf16_bits(q)
    return cache, tables, q, ks, vs


def _sdpa(q, k, v, scale):
    """torch SDPA in fp64: q [H, D], k/v [ctx, H_kv, D] -> [H, D]."""
    tq = torch.from_numpy(q)[None, :, None, :]  # [1, H, 1, D]
    tk = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))[None]  # [1, H_kv, ctx, D]
    tv = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))[None]
    out = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, scale=scale, enable_gqa=(q.shape[0] != k.shape[1]))
    return out[0, :, 0, :].numpy()


# ----- pins, written against a pluggable (gather, attend) pair ------------

def pin_library(gather, attend, seed=0, dtype="f32", hk=2, group=2):
    rng = np.random.default_rng(seed)
    ctxs = [1, 5, 16, 17, 40]
    h, d, bs = hk * group, 8, 16
    cache, tables, q, _, _ = _paged_setup(rng, ctxs, h, hk, d, bs, dtype)
    scale = 1.0 / math.sqrt(d)
    for i, c in enumerate(ctxs):
        k, v = gather(cache, tables[i], c)
        got = attend(att.widen(q[i], dtype), k, v, scale)
        ref = _sdpa(att.widen(q[i], dtype), k, v, scale)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def pin_closed_forms(gather, attend, seed=1):
    rng = np.random.default_rng(seed)
    hk, group, d, bs = 2, 2, 8, 4
    h = hk * group
    scale = 0.37
    q = rng.standard_normal((h, d))
    # identical keys -> mean of V
    for ctx in (1, 3, 9):
        k = np.repeat(rng.standard_normal((1, hk, d)), ctx, axis=0)
        v = rng.standard_normal((ctx, hk, d))
        out = attend(q, k, v, scale)
        for hh in range(h):
            np.testing.assert_allclose(out[hh], v[:, hh // group].mean(axis=0), atol=1e-12, rtol=0)
    # q = 0 -> mean of V
    k = rng.standard_normal((7, hk, d))
    v = rng.standard_normal((7, hk, d))
    out = attend(np.zeros((h, d)), k, v, scale)
    for hh in range(h):
        np.testing.assert_allclose(out[hh], v[:, hh // group].mean(axis=0), atol=1e-12, rtol=0)
    # ctx = 1 -> v exactly
    k1, v1 = rng.standard_normal((1, hk, d)), rng.standard_normal((1, hk, d))
    out = attend(q, k1, v1, scale)
    for hh in range(h):
        assert np.array_equal(out[hh], v1[0, hh // group])
    # constant V -> that constant
    vc = np.full((11, hk, d), 2.5)
    out = attend(q, rng.standard_normal((11, hk, d)), vc, scale)
    np.testing.assert_allclose(out, 2.5, atol=1e-12, rtol=0)
    # one logit 50 above the rest -> its v
    kd = np.zeros((6, hk, d))
    qd = np.zeros((h, d))
    qd[:, 0] = 1.0
    kd[4, :, 0] = 50.0 / scale
    vd = rng.standard_normal((6, hk, d))
    out = attend(qd, kd, vd, scale)
    for hh in range(h):
        np.testing.assert_allclose(out[hh], vd[4, hh // group], atol=1e-12, rtol=0)
    # paged walk: the gather must return the written tokens in logical order
    ctxs = [bs + 3, 2 * bs]
    cache, tables, qq, ks, vs = _paged_setup(rng, ctxs, h, hk, d, bs, "f32", spare=5)
    for i, c in enumerate(ctxs):
        kg, vg = gather(cache, tables[i], c)
        assert np.array_equal(kg, ks[i]) and np.array_equal(vg, vs[i])


def pin_brute_force(gather, attend, seed=2):
    rng = np.random.default_rng(seed)
    for ctx in (1, 2, 3, 4):
        for hk, group in ((1, 1), (2, 1), (1, 2), (2, 2)):
            h, d = hk * group, 3
            q = rng.standard_normal((h, d))
            k = rng.standard_normal((ctx, hk, d))
            v = rng.standard_normal((ctx, hk, d))
            scale = 0.61
            out = attend(q, k, v, scale)
            for hh in range(h):
                g = hh // group
                s = [scale * sum(q[hh][j] * k[t][g][j] for j in range(d)) for t in range(ctx)]
                e = [math.exp(x) for x in s]
                z = sum(e)
                for j in range(d):
                    ref = sum(e[t] / z * v[t][g][j] for t in range(ctx))
                    assert abs(out[hh][j] - ref) < 1e-12


PINS = [pin_library, pin_closed_forms, pin_brute_force]


@pytest.mark.parametrize("pin", PINS)
def test_oracle_pins(pin):
    pin(att.gather_sequence, att.attend_contiguous)


def test_library_pin_bf16():
    pin_library(att.gather_sequence, att.attend_contiguous, seed=3, dtype="bf16", hk=3, group=1)
    pin_library(att.gather_sequence, att.attend_contiguous, seed=4, dtype="bf16", hk=1, group=4)


def test_permutation_invariance_is_bitwise():
    rng = np.random.default_rng(7)
    ctxs = [3, 16, 33, 47]
    hk, group, d, bs = 2, 2, 16, 16
    cache, tables, q, ks, vs = _paged_setup(rng, ctxs, hk * group, hk, d, bs, "bf16", spare=6)
    out1 = att.paged_decode(q, cache, tables, ctxs, 0.25)
    # move every block to a new physical location
    nb = cache.num_blocks
    perm = rng.permutation(nb)
    cache2 = PagedKVCache(nb, hk, d, bs, "bf16")
    cache2.copy_blocks([])
    for b in cache.blocks():
        nb_ = int(perm[b])
        kp, vp, wr = cache2._page(nb_)
        kp[...] = cache.k_page(b)
        vp[...] = cache.v_page(b)
        wr[...] = cache.written(b)
    tables2 = [[int(perm[b]) for b in t] for t in tables]
    out2 = att.paged_decode(q, cache2, tables2, ctxs, 0.25)
    assert np.array_equal(out1, out2)


def test_zero_context_gives_zero_row():
    rng = np.random.default_rng(8)
    cache, tables, q, _, _ = _paged_setup(rng, [5], 2, 2, 4, 4, "f32")
    out = att.paged_decode(np.concatenate([q, q]), cache, [tables[0], []], [5, 0], 0.5)
    assert np.all(out[1] == 0) and np.any(out[0] != 0)


def test_paged_decode_rows_matches_full():
    rng = np.random.default_rng(9)
    ctxs = [4, 20, 1]
    cache, tables, q, _, _ = _paged_setup(rng, ctxs, 4, 2, 8, 4, "f32")
    full = att.paged_decode(q, cache, tables, ctxs, 0.3)
    rows = att.paged_decode_rows(q, cache, tables, ctxs, 0.3, [2, 0])
    assert np.array_equal(rows[0], full[0]) and np.array_equal(rows[2], full[2])


@pytest.mark.parametrize("ctx,part", [(1, 512), (511, 512), (512, 512), (513, 512), (2000, 512), (100, 16), (37, 5)])
def test_lse_merge_equals_unsplit(ctx, part):
    rng = np.random.default_rng(ctx + part)
    hk, group, d = 2, 2, 16
    q = rng.standard_normal((hk * group, d))
    k = rng.standard_normal((ctx, hk, d)) * 3
    v = rng.standard_normal((ctx, hk, d))
    o, lse = att.partition_partials(q, k, v, 0.2, part)
    assert o.shape[0] == -(-ctx // part)
    merged = att.lse_merge(o, lse)
    np.testing.assert_allclose(merged, att.attend_contiguous(q, k, v, 0.2), atol=1e-12, rtol=0)
    # a partition with no tokens (lse = -inf) carries no weight
    o2 = np.concatenate([o, rng.standard_normal((1,) + o.shape[1:])])
    lse2 = np.concatenate([lse, np.full((1, lse.shape[1]), -np.inf)])
    np.testing.assert_allclose(att.lse_merge(o2, lse2), merged, atol=1e-15, rtol=0)


def test_lse_partials_closed_form():
    """One partition: lse = log sum exp(s) and o = the full result."""
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 4))
    k = rng.standard_normal((9, 1, 4))
    v = rng.standard_normal((9, 1, 4))
    o, lse = att.partition_partials(q, k, v, 1.0, 64)
    s = k[:, 0, :] @ q[0]
    assert abs(lse[0, 0] - math.log(sum(math.exp(x) for x in s))) < 1e-12


# ----- planted mistakes: each must be caught by at least one pin ----------

def _mut_head_map(q, k, v, scale):
    h_q, d = q.shape
    ctx, h_kv, _ = k.shape
    out = np.zeros((h_q, d))
    for h in range(h_q):
        g = h % h_kv
        s = scale * (k[:, g, :] @ q[h])
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ v[:, g, :]
    return out


def _mut_no_scale(q, k, v, scale):
    return att.attend_contiguous(q, k, v, 1.0)


def _mut_drop_last(q, k, v, scale):
    if k.shape[0] <= 1:
        return att.attend_contiguous(q, k, v, scale)
    return att.attend_contiguous(q, k[:-1], v[:-1], scale)


def _mut_transposed_kv(q, k, v, scale):
    return att.attend_contiguous(q, v, k, scale)


def _mut_gather_offset(cache, table, ctx):
    """Reads offset (t + 1) % bs of the right block."""
    k, v = att.gather_sequence(cache, table, ctx)
    bs = cache.block_size
    idx = np.array([(t // bs) * bs + ((t % bs) + 1) % min(bs, ctx - (t // bs) * bs) for t in range(ctx)])
    return k[idx], v[idx]


@pytest.mark.parametrize("attend,gather", [
    (_mut_head_map, att.gather_sequence),
    (_mut_no_scale, att.gather_sequence),
    (_mut_drop_last, att.gather_sequence),
    (_mut_transposed_kv, att.gather_sequence),
    (att.attend_contiguous, _mut_gather_offset),
])
def test_pins_catch_planted_mistakes(attend, gather):
    caught = 0
    for pin in PINS:
        try:
            pin(gather, attend)
        except AssertionError:
            caught += 1
    assert caught >= 1
