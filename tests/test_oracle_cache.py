"""Pins for the oracle cache write and block copy, and the workload replay.

* page size: one block holds BLOCK_SIZE tokens of one head — 2048 elements
  per block per head at block size 16, head size 128 (gitcode repo
  walkthrough, section 2.1; tests/golden/page_size.json);
* round trip: reading each written slot back returns the written bytes;
* copy-on-write copy: the destination block equals the source bit for bit;
* replaying a sampling workload, every sequence reads back exactly the
  token values of its own logical history (prompt then its own samples).
"""

import json
import os

import numpy as np
import pytest

from oracle.attention import gather_sequence, widen
from oracle.cache import PagedKVCache
from oracle.replay import block_table_array, replay
from workloads import make_plan, seq_token_sources, stream_kv, to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_page_size_matches_pages():
    with open(os.path.join(GOLDEN, "page_size.json")) as f:
        g = json.load(f)
    c = PagedKVCache(2, 1, g["head_size"], g["block_size"], "bf16")
    assert c.k_page(0)[0].size == g["elements_per_block_per_head"]


def test_write_round_trip_and_skip():
    rng = np.random.default_rng(0)
    c = PagedKVCache(6, 3, 8, 4, "bf16")
    k = to_bf16_bits(rng.standard_normal((7, 3, 8)).astype(np.float32))
    v = to_bf16_bits(rng.standard_normal((7, 3, 8)).astype(np.float32))
    slots = [5, 0, -1, 23, 12, 13, 6]
    c.write(slots, k, v)
    for t, s in enumerate(slots):
        if s == -1:
            continue
        kk, vv = c.read_token(s)
        assert np.array_equal(kk, k[t]) and np.array_equal(vv, v[t])
    with pytest.raises(IndexError):
        c.read_token(1)  # never written
    with pytest.raises(IndexError):
        c.write([24], k[:1], v[:1])  # block 6 is outside the pool


def test_copy_blocks_bitwise():
    rng = np.random.default_rng(1)
    c = PagedKVCache(4, 2, 4, 4, "f32")
    k = rng.standard_normal((3, 2, 4)).astype(np.float32)
    c.write([4, 5, 6], k, -k)
    c.copy_blocks([(1, 3)])
    assert np.array_equal(c.k_page(3), c.k_page(1)) and np.array_equal(c.v_page(3), c.v_page(1))
    assert np.array_equal(c.written(3), c.written(1))


def test_sampling_replay_reads_back_logical_history():
    plan = make_plan("parallel_sampling_13b")
    # shrink: keep the first 3 prompts' requests only (seq ids < 12)
    plan.setup_ops = [op for op in plan.setup_ops
                      if getattr(op, "seq", getattr(op, "parent", 0)) < 12]
    alloc, cache, log = replay(plan)
    n_cow = sum(len(c) for _, _, c in log.appends)
    assert n_cow > 0
    runs = seq_token_sources(plan)
    for sid in range(12):
        parts_k, parts_v = [], []
        for stream, start, n in runs[sid]:
            k, v = stream_kv(plan, stream, start, n)
            parts_k.append(k)
            parts_v.append(v)
        k_ref = widen(np.concatenate(parts_k), "bf16")
        v_ref = widen(np.concatenate(parts_v), "bf16")
        ctx = alloc.length(sid)
        assert ctx == k_ref.shape[0]
        kg, vg = gather_sequence(cache, alloc.block_table(sid), ctx)
        assert np.array_equal(kg, k_ref) and np.array_equal(vg, v_ref)
    # samples of one prompt share the prompt's full blocks
    t0, t1 = alloc.block_table(0), alloc.block_table(1)
    shared = alloc.length(0) - 64  # at least this many prompt tokens
    assert t0[: max(0, shared // 16 - 1)] == t1[: max(0, shared // 16 - 1)]


def test_tiny_replay_tables():
    plan = make_plan("tiny_fp32")
    alloc, cache, log = replay(plan)
    bt = block_table_array(alloc, plan.batch, plan.max_blocks_per_seq)
    assert bt.shape == (4, 7)
    used = sorted(int(b) for b in bt.reshape(-1) if b >= 0)
    assert len(used) == 13 and len(set(used)) == 13
    # blocks are handed out in the seeded permuted order
    assert used == sorted(plan.free_order[:13].tolist())
