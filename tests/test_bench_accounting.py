"""The benchmark's algorithmic work counts, checked on CPU against brute
force over the seeded plans: the decode step's bytes (every context token's
K and V in the cache's element size, query and output, block-table entries,
context lengths; the cache write reads the new tokens' K/V and writes them)
and the chunked-prefill FLOPs (each new token at position p attends p + 1
keys in every query head: 2 D flops for QK^T and 2 D for PV per key)."""

import numpy as np
import pytest

import bench
from workloads import AppendOp, make_plan


@pytest.mark.parametrize("name", ["tiny_fp32", "llama7b_bs64", "gqa_bs256_fp8"])
def test_decode_step_bytes_brute_force(name):
    plan = make_plan(name)
    w = plan.workload
    got = bench.step_bytes(plan)
    kv = 0
    tables = 0
    for c in plan.context_lens.tolist():
        for _t in range(int(c)):
            kv += 2 * w.num_kv_heads * w.head_size * w.cache_elem_bytes
        tables += 4 * len(range(0, int(c), w.block_size))
    qo = 2 * plan.B * w.num_heads * w.head_size * w.elem_bytes
    assert got["kv"] == kv
    assert got["decode"] == kv + qo + tables + 4 * plan.B
    new_tokens = sum(op.n for op in plan.step_ops if isinstance(op, AppendOp))
    assert new_tokens == len(plan.step_ops)  # one token per sequence in a decode step
    per_token = w.num_kv_heads * w.head_size * 2 * (w.elem_bytes + w.cache_elem_bytes) + 8
    assert got["write"] == new_tokens * per_token
    assert got["step"] == got["decode"] + got["write"]


def test_shared_prefix_unique_bytes_brute_force():
    """The sampling workload under a shared-prefix decode: the unique KV
    bytes are the distinct (physical block, kv head, slot) entries the step
    attends, found by replaying the requests on the oracle allocator and
    walking every sequence's table; the groups come from the oracle's model
    of the grouping rule."""
    from oracle.cascade import prefix_groups
    from oracle.replay import replay

    plan = make_plan("parallel_sampling_13b")
    w = plan.workload
    alloc, _, _ = replay(plan, write_values=False)
    tables = [alloc.block_table(int(s)) for s in plan.batch]
    lens = [int(c) for c in plan.context_lens]
    gs, gb = prefix_groups(tables, lens, 4, w.block_size)
    assert all(b > 0 for b in gb)
    got = bench.step_bytes(plan, (np.array(gs), np.array(gb)))
    read = set()
    for t, c in zip(tables, lens):
        for pos in range(c):
            read.add((t[pos // w.block_size], pos % w.block_size))
    per_slot = 2 * w.num_kv_heads * w.head_size * w.cache_elem_bytes
    assert got["kv"] == len(read) * per_slot
    assert got["kv_logical"] == sum(lens) * per_slot
    assert got["kv"] < got["kv_logical"] / 3


@pytest.mark.parametrize("name", ["prefill_tiny", "prefill_mixed_gqa"])
def test_prefill_flops_brute_force(name):
    plan = make_plan(name)
    w = plan.workload
    total = 0
    for c, n in zip(plan.context_lens.tolist(), plan.query_lens.tolist()):
        for j in range(n):
            pos = c - n + j
            total += w.num_heads * (pos + 1) * 4 * w.head_size
    assert bench.prefill_flops(plan) == total
    assert bench.is_prefill(plan)
    assert not bench.is_prefill(make_plan("llama7b_bs64"))


def test_aggregate_value_scales_with_ranks():
    assert bench.aggregate_value(1e9, 1.0, 1) == pytest.approx(1000.0)
    assert bench.aggregate_value(1e9, 1.0, 4) == pytest.approx(4000.0)
    assert np.allclose(bench.max_over_ranks([1.0, 2.5], None, 1), [1.0, 2.5])


def test_step_kv_shapes():
    """The step's new-token K/V: one row per appended token, empty for a
    step that appends nothing (all requests made before the step)."""
    for name, rows in (("llama7b_bs64", 64), ("prefill_tiny", None), ("parallel_sampling_13b", 0)):
        plan = make_plan(name)
        w = plan.workload
        k, v = bench.step_kv(plan)
        n = sum(op.n for op in plan.step_ops)
        assert k.shape == v.shape == (n, w.num_kv_heads, w.head_size)
        if rows is not None:
            assert n == rows


@pytest.mark.parametrize("name,unit", [("tiny_fp32", "GB/s"), ("prefill_tiny", "TFLOP/s")])
def test_reference_arm_prints_the_contract_line(name, unit):
    """`bench.py --impl reference` times the oracle on the host and prints one
    JSON line with the contract's keys (CPU only)."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", name,
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the oracle is timed once, by rank 0; any other rank
    exits 0 at once and prints nothing."""
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=root,
                         env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    assert not [l for l in res.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("name", ["tiny_fp32", "llama7b_bs64", "parallel_sampling_13b", "prefill_mixed_gqa"])
def test_allocator_report_matches_the_oracle_replay(name):
    """The benchmark's memory report (blocks in use, unused slots, tokens
    held, copy-on-write copies) equals the oracle block manager's on the same
    requests; only last blocks waste (at most bs - 1 slots per sequence); in
    the sampling workload every prompt whose length is not a multiple of the
    block size costs 3 copies (4 samples write into its shared last block)."""
    from oracle.allocator import BlockAllocator
    from workloads import AddOp, ForkOp

    plan = make_plan(name)
    w = plan.workload
    rep = bench.allocator_report(plan)
    o = BlockAllocator(plan.num_blocks, w.block_size, plan.free_order)
    cows = 0
    for op in list(plan.setup_ops) + list(plan.step_ops):
        if isinstance(op, AddOp):
            o.add(op.seq)
        elif isinstance(op, ForkOp):
            o.fork(op.parent, op.child)
        else:
            cows += len(o.append(op.seq, op.n)[1])
    used = plan.num_blocks - o.num_free()
    held = sum(o.length(s) for s in o.sequences())
    longest = max(int(c) for c in plan.context_lens)
    assert rep == {"blocks_used": used, "waste_slots": o.waste_slots(),
                   "waste_frac": round(o.waste_slots() / (used * w.block_size), 5), "tokens_held": held,
                   "cow_copies": cows,
                   "waste_frac_if_contiguous": round(1.0 - held / (len(o.sequences()) * longest), 5)}
    assert rep["waste_slots"] <= (w.block_size - 1) * len(o.sequences())
    if name == "parallel_sampling_13b":
        from workloads.synth import parallel_sampling_lengths

        plen, _ = parallel_sampling_lengths(w)
        assert rep["cow_copies"] == 3 * sum(1 for n in plen.tolist() if n % w.block_size)


def test_prefill_row_requests_reproduce_the_whole_request():
    """The reference arm times the prefill oracle on runs of consecutive new
    tokens, each asked as the request that ends at the run's last token.
    Causal attention makes those rows equal to the whole request's (up to
    fp64 summation order), and the runs' FLOPs add up to the step's."""
    import numpy as np

    from oracle.prefill import paged_prefill_seqs

    plan = make_plan("prefill_tiny")
    st = bench.oracle_state(plan)
    scale = 1.0 / np.sqrt(plan.workload.head_size)
    whole = paged_prefill_seqs(st["q"], st["cache"], st["tables"], plan.context_lens, plan.query_start, scale,
                               range(plan.B))
    total = 0
    for i in range(plan.B):
        n = int(plan.query_lens[i])
        for j0 in range(0, n, 5):
            j1 = min(n, j0 + 5)
            q, tables, cl, qs = bench.prefill_row_request(plan, st, i, j0, j1)
            part = paged_prefill_seqs(q, st["cache"], tables, cl, qs, scale, [0])[0]
            # the same rows; only fp64 summation order differs (shorter masked key range)
            assert np.max(np.abs(part - whole[i][j0:j1]), initial=0.0) <= 1e-12, (i, j0)
            total += bench.prefill_rows_flops(plan, i, j0, j1)
    assert total == bench.prefill_flops(plan)


@pytest.mark.parametrize("name", ["tiny_fp32", "prefill_tiny"])
def test_reference_arm_bounds_each_step(name):
    """Many steps stay within the oracle time budget: the oracle's copy of
    the workload is built once and each step is a bounded sample."""
    import json
    import os
    import subprocess
    import sys
    import time

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    t0 = time.time()
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", name,
                          "--steps", "2000", "--warmup", "20", "--ref-seconds", "3"], capture_output=True, text=True,
                         timeout=300, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    assert time.time() - t0 < 120
    d = json.loads([l for l in res.stdout.splitlines() if l.startswith("{")][0])
    assert d["steps"] == 2000 and d["value"] > 0


def test_kernel_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    """The profiles' kernel_source_sha: rewording a comment or re-spacing keeps
    the hash, any code change (including inside an inline-PTX string) does
    not, and a '//' inside a string literal is code."""
    csrc = tmp_path / "paged_kv_cache_351_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))

    def h(text):
        (csrc / "k.cuh").write_text(text)
        return bench.kernel_source_hash(("k.cuh",))

    base = h('int f(int x) {  // add one\n  /* block\n comment */ return x + 1;\n}\nconst char* s = "a//b";\n')
    assert h('int f(int x) {  // add ONE, reworded\n  return   x + 1;\n}\nconst char* s = "a//b";\n') == base
    assert h('int f(int x) {\n  return x + 2;\n}\nconst char* s = "a//b";\n') != base
    assert h('int f(int x) {\n  return x + 1;\n}\nconst char* s = "a//c";\n') != base
    assert h('int f(int x) {\n  return x + 1;\n}\nconst char* s = "a";\n') != base
