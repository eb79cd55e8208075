"""Pins for the shared-prefix decode's oracle (oracle.cascade) and for the
library's host grouping (pa_alloc_prefix_groups) against it.

* cascade_decode_rows — a shared-prefix partial and a suffix partial merged
  by log-sum-exp — equals the plain definition of attention
  (attention.paged_decode) to 1e-12, for any grouping whose members hold the
  same leading blocks (the pages: parallel samples share the prompt's blocks
  and its computation, CSDN discovery note item 2); a planted mistake in the
  split (the suffix starting one token late) is caught.
* prefix_groups: the hand-worked example in tests/golden; on random fork
  forests the groups tile the batch, respect the size limit, and every
  member holds the group's shared blocks (full blocks, same ids, same
  indices); the C++ allocator's grouping equals the model.
"""

import json
import math
import os

import numpy as np
import pytest

import paged_kv_cache_351_b200 as pa
from oracle import attention as att
from oracle.allocator import BlockAllocator
from oracle.cache import PagedKVCache
from oracle.cascade import cascade_decode_rows, prefix_groups

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "prefix_groups_example.json")
BS = 16


def _forest(rng, n_prompts, max_samples, hk, d, dtype="f32", forks_of_forks=False, shuffle=False):
    """Prompts forked into samples that append their own tokens, on the
    oracle allocator and the C++ allocator in lockstep; K/V written into an
    oracle cache.  Returns (oracle alloc, C++ alloc, cache, batch ids)."""
    lens = rng.integers(1, 200, size=n_prompts)
    nb = int(sum(-(-int(l) // BS) for l in lens) * max_samples * 2 + 64)
    order = rng.permutation(nb).astype(np.int32)
    ao = BlockAllocator(nb, BS, order)
    ac = pa.Allocator(nb, BS, order)
    cache = PagedKVCache(nb, hk, d, BS, dtype)

    def append(seq, n):
        slots_o, cow_o = ao.append(seq, n)
        slots_c, cow_c = ac.append(seq, n)
        assert list(slots_c) == list(slots_o) and cow_c == cow_o
        cache.copy_blocks(cow_o)
        if n:
            cache.write(slots_o, rng.standard_normal((n, hk, d)).astype(np.float32),
                        rng.standard_normal((n, hk, d)).astype(np.float32))

    batch, sid = [], 0
    for p in range(n_prompts):
        root = sid
        sid += 1
        ao.add(root)
        ac.add(root)
        append(root, int(lens[p]))
        members = [root]
        for _ in range(int(rng.integers(0, max_samples))):
            parent = members[int(rng.integers(0, len(members)))] if forks_of_forks else root
            ao.fork(parent, sid)
            ac.fork(parent, sid)
            members.append(sid)
            sid += 1
            if forks_of_forks:
                append(sid - 1, int(rng.integers(0, 40)))
        for m in members:
            append(m, int(rng.integers(0, 40)))
        batch += members
    if shuffle:
        rng.shuffle(batch)
    return ao, ac, cache, batch


def test_golden_example():
    with open(GOLDEN) as f:
        g = json.load(f)
    gs, gb = prefix_groups(g["tables"], g["lens"], g["max_group_size"], g["block_size"])
    assert gs == g["group_start"] and gb == g["group_blocks"]


@pytest.mark.parametrize("seed", range(6))
def test_groups_are_valid(seed):
    rng = np.random.default_rng(100 + seed)
    ao, _, _, batch = _forest(rng, 12, 6, 1, 4, forks_of_forks=seed % 2 == 1, shuffle=seed >= 4)
    tables = [ao.block_table(s) for s in batch]
    lens = [ao.length(s) for s in batch]
    for mg in (1, 2, 4, 8):
        gs, gb = prefix_groups(tables, lens, mg, BS)
        assert gs[0] == 0 and gs[-1] == len(batch) and all(a < b for a, b in zip(gs, gs[1:]))
        for v, shared in enumerate(gb):
            members = range(gs[v], gs[v + 1])
            assert len(members) <= mg
            if len(members) == 1:
                assert shared == 0
            for i in members:
                assert shared * BS <= lens[i]
                assert tables[i][:shared] == tables[gs[v]][:shared]


@pytest.mark.parametrize("seed", range(6))
def test_library_grouping_matches_model(seed):
    rng = np.random.default_rng(200 + seed)
    ao, ac, _, batch = _forest(rng, 10, 8, 1, 4, forks_of_forks=seed % 2 == 1, shuffle=seed >= 4)
    tables = [ao.block_table(s) for s in batch]
    lens = [ao.length(s) for s in batch]
    for mg in (1, 2, 3, 4, 8):
        gs, gb = prefix_groups(tables, lens, mg, BS)
        cgs, cgb = ac.prefix_groups(batch, mg)
        assert list(cgs) == gs and list(cgb) == gb, mg


def test_library_grouping_errors():
    a = pa.Allocator(8, BS)
    a.add(1)
    with pytest.raises(pa.PagedAttentionError):
        a.prefix_groups([1, 2], 4)  # unknown sequence
    with pytest.raises(pa.PagedAttentionError):
        a.prefix_groups([1], 0)  # no room for a member
    gs, gb = a.prefix_groups([], 4)
    assert list(gs) == [0] and len(gb) == 0


def _random_grouping(rng, tables, lens, max_size):
    """Any valid grouping: random run lengths, shared count anywhere from 0
    to the members' common full blocks."""
    n, gs, gb, k = len(tables), [], [], 0
    while k < n:
        size = int(rng.integers(1, max_size + 1))
        members = list(range(k, min(n, k + size)))
        common = min(lens[i] for i in members) // BS
        c = 0
        while c < common and all(tables[i][c] == tables[k][c] for i in members):
            c += 1
        gs.append(k)
        gb.append(int(rng.integers(0, c + 1)))
        k = members[-1] + 1
    gs.append(n)
    return gs, gb


@pytest.mark.parametrize("seed", range(5))
def test_cascade_equals_plain_attention(seed):
    rng = np.random.default_rng(300 + seed)
    hk, g, d = 2, 2, 8
    ao, _, cache, batch = _forest(rng, 8, 5, hk, d, forks_of_forks=seed % 2 == 1)
    tables = [ao.block_table(s) for s in batch]
    lens = [ao.length(s) for s in batch]
    q = rng.standard_normal((len(batch), hk * g, d)).astype(np.float32)
    scale = 1 / math.sqrt(d)
    plain = att.paged_decode(q, cache, tables, lens, scale)
    for gs, gb in (prefix_groups(tables, lens, 4, BS), _random_grouping(rng, tables, lens, 6)):
        got = cascade_decode_rows(q, cache, tables, lens, gs, gb, scale)
        for i in range(len(batch)):
            assert np.max(np.abs(got[i] - plain[i])) <= 1e-12


def test_cascade_catches_a_shifted_suffix():
    """A split whose suffix starts one token late drops a token: caught."""
    rng = np.random.default_rng(7)
    ao, _, cache, batch = _forest(rng, 4, 4, 1, 8)
    tables = [ao.block_table(s) for s in batch]
    lens = [ao.length(s) for s in batch]
    q = rng.standard_normal((len(batch), 1, 8)).astype(np.float32)
    gs, gb = prefix_groups(tables, lens, 4, BS)
    assert any(b > 0 for b in gb)
    plain = att.paged_decode(q, cache, tables, lens, 0.3)
    i = next(i for v, b in enumerate(gb) if b > 0 for i in range(gs[v], gs[v + 1]) if lens[i] > b * BS + 1)
    v = max(u for u in range(len(gb)) if gs[u] <= i)
    p = gb[v] * BS
    qi = att.widen(q[i], "f32")
    k, vv = att.gather_sequence(cache, tables[i], lens[i])
    o1, l1 = att.partition_partials(qi, k[:p], vv[:p], 0.3, p)
    o2, l2 = att.partition_partials(qi, k[p + 1:], vv[p + 1:], 0.3, lens[i] - p - 1)
    wrong = att.lse_merge(np.stack([o1[0], o2[0]]), np.stack([l1[0], l2[0]]))
    assert np.max(np.abs(wrong - plain[i])) > 1e-6
