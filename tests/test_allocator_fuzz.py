"""Property-based fuzzing of the C++ block allocator against the oracle
(CPU only).  Hypothesis draws request sequences — add, append, fork, free,
prefix-cached add with token ids, swap out and in — over a small device and
host pool; after every request the slots, copy-on-write pairs, swap pairs,
block tables, reference counts and free counts must be identical, and an
out-of-blocks failure must happen on both sides and change nothing.  On a
failure Hypothesis shrinks the sequence to a minimal one."""

import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import paged_kv_cache_351_b200 as pa
from oracle.allocator import BlockAllocator, OutOfBlocks

NB, NH, BS = 12, 8, 4

op = st.one_of(
    st.tuples(st.just("add"), st.integers(0, 10)),
    st.tuples(st.just("prefix"), st.lists(st.integers(0, 1), min_size=1, max_size=11)),
    st.tuples(st.just("append"), st.integers(0, 7), st.integers(1, 6)),
    st.tuples(st.just("fork"), st.integers(0, 7)),
    st.tuples(st.just("free"), st.integers(0, 7)),
    st.tuples(st.just("swap_out"), st.integers(0, 7)),
    st.tuples(st.just("swap_in"), st.integers(0, 7)),
)


def _same_state(c, o, live):
    assert c.num_free() == o.num_free()
    assert c.evictable() == list(o._evictable)
    for b in range(o.num_blocks):
        assert c.refcount(b) == o.refcount(b), b
    for s in live:
        if not o.is_swapped(s):
            assert c.block_table(s) == o.block_table(s), s
        assert c.length(s) == o.length(s), s


def _both(fo, fc):
    try:
        ro = fo()
    except OutOfBlocks:
        with pytest.raises(pa.OutOfBlocksError):
            fc()
        return None
    return ro, fc()


@settings(max_examples=400, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(order=st.permutations(list(range(NB))), horder=st.permutations(list(range(NH))),
       ops=st.lists(op, min_size=1, max_size=60))
def test_allocator_fuzz_matches_oracle(order, horder, ops):
    c, o = pa.Allocator(NB, BS, order), BlockAllocator(NB, BS, order)
    c.set_host_pool(NH, horder)
    o.set_host_pool(NH, horder)
    live, nxt = [], 0
    for item in ops:
        kind = item[0]
        resident = [s for s in live if not o.is_swapped(s)]
        swapped = [s for s in live if o.is_swapped(s)]
        if kind == "add":
            c.add(nxt)
            o.add(nxt)
            live.append(nxt)
            nxt += 1
        elif kind == "prefix":
            toks = item[1]
            assert c.add_prefix(nxt, toks) == o.add_prefix(nxt, toks)
            hit = o.length(nxt)
            live.append(nxt)
            res = _both(lambda: o.append_tokens(nxt, toks[hit:]), lambda: c.append_tokens(nxt, toks[hit:]))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
            nxt += 1
        elif kind == "append" and resident:
            s = resident[item[1] % len(resident)]
            n = item[2]
            res = _both(lambda: o.append(s, n), lambda: c.append(s, n))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
        elif kind == "fork" and resident:
            p = resident[item[1] % len(resident)]
            o.fork(p, nxt)
            c.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif kind == "free" and live:
            s = live.pop(item[1] % len(live))
            o.free(s)
            c.free(s)
        elif kind == "swap_out" and resident:
            s = resident[item[1] % len(resident)]
            res = _both(lambda: o.swap_out(s), lambda: c.swap_out(s))
            if res:
                assert [tuple(p) for p in res[1].tolist()] == res[0]
        elif kind == "swap_in" and swapped:
            s = swapped[item[1] % len(swapped)]
            res = _both(lambda: o.swap_in(s), lambda: c.swap_in(s))
            if res:
                assert [tuple(p) for p in res[1].tolist()] == res[0]
        _same_state(c, o, live)
        o.check_invariants()
    assert c.num_host_free() == o.num_host_free()


# Long prompts over a small alphabet: deep registered chains that branch
# wherever two prompts diverge, so evictions unregister whole subtrees.
deep_op = st.one_of(
    st.tuples(st.just("prefix"), st.lists(st.integers(0, 1), min_size=1, max_size=90)),
    st.tuples(st.just("append"), st.integers(0, 7), st.integers(1, 9)),
    st.tuples(st.just("fork"), st.integers(0, 7)),
    st.tuples(st.just("free"), st.integers(0, 7)),
)


@settings(max_examples=300, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])
@given(order=st.permutations(list(range(48))), ops=st.lists(deep_op, min_size=1, max_size=40))
def test_allocator_fuzz_deep_prefix_trees(order, ops):
    nb, bs = 48, 2
    c, o = pa.Allocator(nb, bs, order), BlockAllocator(nb, bs, order)
    live, nxt = [], 0
    for item in ops:
        kind = item[0]
        if kind == "prefix":
            toks = item[1]
            assert c.add_prefix(nxt, toks) == o.add_prefix(nxt, toks)
            hit = o.length(nxt)
            live.append(nxt)
            res = _both(lambda: o.append_tokens(nxt, toks[hit:]), lambda: c.append_tokens(nxt, toks[hit:]))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
            nxt += 1
        elif kind == "append" and live:
            s = live[item[1] % len(live)]
            toks = [(s + k) % 2 for k in range(item[2])]
            res = _both(lambda: o.append_tokens(s, toks), lambda: c.append_tokens(s, toks))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
        elif kind == "fork" and live:
            p = live[item[1] % len(live)]
            o.fork(p, nxt)
            c.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif kind == "free" and live:
            s = live.pop(item[1] % len(live))
            o.free(s)
            c.free(s)
        _same_state(c, o, live)
        assert c.stats()["num_cached"] == o.num_cached()
        o.check_invariants()
