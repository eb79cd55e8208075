#!/usr/bin/env python
"""Paged decode attention benchmark (one serving step of one attention layer).

Workload: the LLaMA-7B-shaped batch-64 decode (B=64, H=H_kv=32, D=128, bf16
KV, 16-token blocks, lognormal context lengths with median 512 clipped to
[16, 2048], blocks scattered over a 40 GB pool), seeded and synthetic.

A step is the whole hot path for one batch: the new token of every sequence
is written into its slot (pa_reshape_and_cache), then paged decode attention
runs over every sequence's blocks (pa_decode: the decode kernel and, when the
context is split, the log-sum-exp merge).  The allocator's bookkeeping for
the step is done before timing (host-side, no copy-on-write in this
workload).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  value = algorithmic bytes of the step (KV,
query, output, block tables, context lengths, and the cache write's read +
write) / device time per step, summed over ranks; the KV read per step
(0.71 GB) is larger than the 126 MB L2, so no flush is needed.
"""

from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention: KV-read GB/s (% of B200 HBM peak) and decode tok/s"
WORKLOAD = "llama7b_bs64"
PREFILL_METRIC = "chunked-prefill paged attention: TFLOP/s (causal QK^T and PV of every new token)"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--partition", type=int, default=0, help="pa_decode partition_tokens (0 auto, -1 none, >0 fixed)")
    ap.add_argument("--pool-gb", type=float, default=None, help="shrink the block pool (profiling on a small case)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="--impl reference: oracle time spread over the warm-up and timed steps")
    ap.add_argument("--tuning", default="", help="warps,stages,ctas_per_sm for pa_set_decode_tuning")
    ap.add_argument("--cascade", choices=["auto", "on", "off"], default="auto",
                    help="shared-prefix decode (pa_decode_cascade) when forks of one prompt share blocks")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# workload and byte accounting
# ---------------------------------------------------------------------------

def workload_plan(name, pool_gb=None):
    from workloads import make_plan

    plan = make_plan(name)
    if pool_gb is not None:
        import numpy as np

        w = plan.workload
        nb = int(pool_gb * 1e9) // (2 * w.num_kv_heads * w.block_size * w.head_size * w.cache_elem_bytes)
        need = sum(-(-int(c) // w.block_size) for c in plan.context_lens)
        nb = max(nb, need)
        plan.num_blocks = nb
        plan.free_order = np.random.default_rng(plan.workload.seed + 1000).permutation(nb).astype(np.int32)
    return plan


def step_bytes(plan, groups=None):
    """Algorithmic bytes: the decode reads every context token's K and V (in
    the cache's element size), the query and writes the output (in the
    query's), plus block tables and lengths; the write reads the new tokens'
    K/V and writes them into the cache.  With ``groups`` (group_start,
    group_blocks of a shared-prefix decode) a group's shared blocks count
    once, not once per member: ``kv`` is then the unique bytes and
    ``kv_logical`` what a per-sequence decode reads."""
    w = plan.workload
    e, ec, bs = w.elem_bytes, w.cache_elem_bytes, w.block_size
    ctx = [int(c) for c in plan.context_lens]
    per_tok = 2 * w.num_kv_heads * w.head_size * ec
    kv_logical = sum(ctx) * per_tok
    saved_blocks = 0
    if groups is not None:
        gs, gb = groups
        saved_blocks = sum((int(gs[v + 1]) - int(gs[v]) - 1) * int(gb[v]) for v in range(len(gb)))
    kv = kv_logical - saved_blocks * bs * per_tok
    qo = 2 * plan.B * w.num_heads * w.head_size * e
    tables = sum(4 * (-(-c // bs)) for c in ctx) - 4 * saved_blocks
    lens = 4 * plan.B
    decode = kv + qo + tables + lens
    n_new = len(plan.step_ops)
    write = n_new * w.num_kv_heads * w.head_size * 2 * (e + ec) + 8 * n_new
    return {"kv": kv, "kv_logical": kv_logical, "decode": decode, "write": write, "step": decode + write}


def allocator_report(plan):
    """Memory use of the workload's paged cache after its step: the
    workload's requests (setup and step) replayed on a fresh host block
    allocator of the library.  Blocks in use, the slots they leave unused
    (only a sequence's last block can hold any), that waste as a fraction of
    the slots in use, tokens held per sequence (shared prompt tokens counted
    once per holder) and the copy-on-write copies the requests caused.  For
    comparison, the fraction of slots a contiguous layout would leave unused
    if every sequence reserved the batch's longest context (no sharing)."""
    import paged_kv_cache_351_b200 as pa
    from workloads import AddOp, ForkOp

    w = plan.workload
    alloc = pa.Allocator(plan.num_blocks, w.block_size, plan.free_order)
    cows = 0
    for op in list(plan.setup_ops) + list(plan.step_ops):
        if isinstance(op, AddOp):
            alloc.add(op.seq)
        elif isinstance(op, ForkOp):
            alloc.fork(op.parent, op.child)
        else:
            cows += len(alloc.append(op.seq, op.n)[1])
    st = alloc.stats()
    used = st["num_blocks"] - st["num_free"]
    reserved = st["num_seqs"] * max([int(c) for c in plan.context_lens] + [1])
    return {"blocks_used": used, "waste_slots": st["waste_slots"],
            "waste_frac": round(st["waste_slots"] / max(1, used * w.block_size), 5),
            "tokens_held": st["num_tokens"], "cow_copies": cows,
            "waste_frac_if_contiguous": round(1.0 - st["num_tokens"] / reserved, 5)}


def is_prefill(plan):
    """A multi-token step (some sequence brings more than one new token)."""
    return bool((plan.query_lens != 1).any())


def prefill_flops(plan):
    """Algorithmic FLOPs of one multi-token step: the new token at position p
    of a sequence attends p + 1 keys in every query head, 2 * D flops for its
    QK^T dot product and 2 * D for its share of P V per key."""
    w = plan.workload
    total = 0
    for c, n in zip(plan.context_lens.tolist(), plan.query_lens.tolist()):
        prior = c - n
        total += n * prior + n * (n + 1) // 2
    return 4 * w.head_size * w.num_heads * total


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor peak (burst: the prefill kernel is timed alone)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|//[^\n]*|/\*.*?\*/', re.S)


def kernel_source_hash(files=("pa_decode.cuh", "pa_common.cuh")):
    """Hash of a kernel's source files with comments removed and blank
    space collapsed: it changes when the code does, not when a comment is
    reworded (string literals, such as inline PTX, are kept)."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_351_b200", "csrc", f)) as fh:
            text = fh.read()
        code = _CODE_TOKENS.sub(lambda m: m.group(0) if m.group(0).startswith('"') else " ", text)
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


PREFILL_SOURCES = ("pa_prefill.cuh", "pa_tc.cuh", "pa_common.cuh")


def ncu_traffic(workload, kernel="decode_kernel", files=("pa_decode.cuh", "pa_common.cuh")):
    """DRAM bytes (read + write) per launch of a kernel from the committed
    ncu summary of this workload, if it was taken on the current kernel
    source; else None."""
    p = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        vals = {}
        with open(p) as f:
            for line in f:
                k, _, v = line.strip().partition(":")
                if k in ("workload", "kernel_source_sha", "dram_bytes_per_launch"):
                    vals[k] = v.strip()
        if vals.get("kernel_source_sha") != kernel_source_hash(files) or vals.get("workload") != workload:
            return None
        return float(vals["dram_bytes_per_launch"])
    except Exception:
        return None


def profile_key(name, partition, shared, groupable):
    """Workload key of the ncu summary that matches the launch bench times:
    the workload name, plus the partition size in fixed-partition mode, plus
    "_no_prefix_groups" when a workload with shared prompts is decoded
    without the shared-prefix path."""
    key = name if partition <= 0 else f"{name}_{partition}"
    return key + "_no_prefix_groups" if groupable and not shared else key


def max_over_ranks(values, device, world):
    """Each rank's device-timed values -> their maximum over all ranks (the
    job is as slow as its slowest replica)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def warm(step, stream, warmup, min_busy_s=0.05):
    """Untimed warm-up: at least max(3, warmup) steps, continued in bursts
    until the GPU has been kept busy for min_busy_s of wall time, then a
    synchronize."""
    import torch

    t0 = time.perf_counter()
    n = 0
    with torch.cuda.stream(stream):
        while n < max(3, warmup) or time.perf_counter() - t0 < min_busy_s:
            for _ in range(max(3, warmup)):
                step()
            n += max(3, warmup)
            torch.cuda.synchronize()


def aggregate_value(bytes_per_step, ms_per_step, world):
    """Whole-job GB/s: every replica moves bytes_per_step per step; the step
    time is the max over ranks."""
    return bytes_per_step * world / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------------------
# device setup through the library
# ---------------------------------------------------------------------------

def step_kv(plan):
    """K and V (storage form, [new tokens, H_kv, D]) of the step's new tokens,
    request by request; empty arrays when the step appends nothing."""
    import numpy as np

    from workloads import stream_kv

    w = plan.workload
    parts = [stream_kv(plan, op.stream, op.start, op.n) for op in plan.step_ops]
    if not parts:
        empty = np.zeros((0, w.num_kv_heads, w.head_size), np.float32 if w.dtype == "f32" else np.uint16)
        return empty, empty.copy()
    return np.concatenate([k for k, _ in parts]), np.concatenate([v for _, v in parts])


def setup_device(plan, device):
    """Replay the workload's setup requests through the host allocator and
    the library's copy/write kernels; return the runtime and the step's
    inputs (slots, new K/V, query, block tables, context lengths)."""
    import numpy as np
    import torch

    from paged_kv_cache_351_b200.runtime import PagedKVCacheGPU
    from workloads import AddOp, AppendOp, ForkOp, kv_scales, query_values, stream_kv

    w = plan.workload
    tdt = torch.float32 if w.dtype == "f32" else torch.bfloat16  # query/output and new-token type

    def dev(raw):
        if w.dtype == "f32":
            return torch.from_numpy(np.ascontiguousarray(raw)).to(device)
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).to(device).view(torch.bfloat16)

    scales = kv_scales(plan) if w.cache_dtype == "fp8" else (None, None)
    kv = PagedKVCacheGPU(plan.num_blocks, w.num_kv_heads, w.head_size, w.cache_dtype, w.block_size,
                         plan.free_order, device=device, k_scale=scales[0], v_scale=scales[1])
    pend = {"seqs": set(), "slots": [], "k": [], "v": [], "pairs": []}

    def flush():
        if pend["slots"]:
            pairs = (torch.from_numpy(np.concatenate(pend["pairs"])).to(device) if pend["pairs"] else None)
            kv.write(torch.from_numpy(np.concatenate(pend["slots"])).to(device), dev(np.concatenate(pend["k"])),
                     dev(np.concatenate(pend["v"])), pairs)
        pend["seqs"].clear(), pend["slots"].clear(), pend["k"].clear(), pend["v"].clear(), pend["pairs"].clear()

    for op in plan.setup_ops:
        if isinstance(op, AddOp):
            kv.add(op.seq)  # a new sequence touches no pending block
        elif isinstance(op, ForkOp):
            flush()
            kv.fork(op.parent, op.child)
        else:
            if op.seq in pend["seqs"]:
                flush()
            slots, pairs = kv.append([op.seq], [op.n])
            k, v = stream_kv(plan, op.stream, op.start, op.n)
            pend["seqs"].add(op.seq)
            pend["slots"].append(slots)
            pend["k"].append(k)
            pend["v"].append(v)
            if len(pairs):
                pend["pairs"].append(pairs)
            if sum(len(s) for s in pend["slots"]) > 200_000:
                flush()
    flush()
    # the step's allocator work (host): the new tokens of the step (one per
    # sequence for decode, none when every request was made before the step)
    seqs = [op.seq for op in plan.step_ops]
    slots, pairs = kv.append(seqs, [op.n for op in plan.step_ops])
    assert len(pairs) == 0
    key, value = step_kv(plan)
    tables, lens = kv.block_tables(plan.batch, plan.max_blocks_per_seq)
    inputs = {
        "slots": slots, "key": key, "value": value,
        "query": query_values(plan), "tables": tables, "lens": lens, "tdt": tdt, "dev": dev,
    }
    torch.cuda.synchronize()
    return kv, inputs


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid, interval_ms=100):
        self.uuid = uuid
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(interval_ms), "-i", uuid], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# CPU oracle timing
# ---------------------------------------------------------------------------

def oracle_state(plan):
    """The oracle's own copy of the workload, built once and outside every
    timed sample: its allocator and cache replayed from the requests, the
    block tables and the queries; plus where the next sample starts."""
    from oracle.replay import block_table_array, replay
    from workloads import query_values

    alloc, cache, _ = replay(plan)
    return {"cache": cache, "tables": block_table_array(alloc, plan.batch, plan.max_blocks_per_seq),
            "q": query_values(plan), "next": (0, 0)}


def _threads():
    try:
        from threadpoolctl import threadpool_info

        return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        return 1


def oracle_timing(plan, seconds, max_rows=None, state=None):
    """Time the oracle as it stands (fp64 NumPy, walking the block tables)
    on whole rows (one sequence, all heads) of the same workload until
    ``seconds`` have passed (at least one row).  With a ``state`` from
    ``oracle_state`` the rows continue where its previous sample stopped."""
    from oracle.attention import paged_decode_rows

    st = state if state is not None else oracle_state(plan)
    lens = plan.context_lens
    scale = 1.0 / math.sqrt(plan.workload.head_size)
    w = plan.workload
    per_tok = 2 * w.num_kv_heads * w.head_size * w.cache_elem_bytes
    done_bytes, rows_done, i = 0, 0, st["next"][0]
    t0 = time.perf_counter()
    while True:
        paged_decode_rows(st["q"], st["cache"], st["tables"], lens, scale, [i])
        done_bytes += int(lens[i]) * per_tok + 2 * w.num_heads * w.head_size * w.elem_bytes
        rows_done += 1
        i = (i + 1) % plan.B
        el = time.perf_counter() - t0
        if el >= seconds or (max_rows is not None and rows_done >= max_rows):
            break
    st["next"] = (i, 0)
    return {"gbs": done_bytes / el / 1e9, "seconds": el, "rows": rows_done, "cores": _threads(),
            "tok_per_s": rows_done / el}


def _prefix_sum(m):
    return m * (m + 1) // 2


def prefill_rows_flops(plan, i, j0, j1):
    """Causal QK^T and PV FLOPs of new tokens j0 .. j1-1 of sequence i: the
    token at position p attends p + 1 keys in every query head."""
    w = plan.workload
    c = int(plan.context_lens[i]) - int(plan.query_lens[i])
    return 4 * w.head_size * w.num_heads * (_prefix_sum(c + j1) - _prefix_sum(c + j0))


def prefill_row_request(plan, state, i, j0, j1):
    """New tokens j0 .. j1-1 of sequence i as a request of their own: the
    same query rows over the context that ends at token j1 - 1 (causal
    attention gives them the rows of the whole request, up to fp64
    summation order).  Returns
    the oracle's arguments (query, block tables, context lengths,
    query_start) for that one-sequence request."""
    import numpy as np

    a = int(plan.query_start[i])
    c = int(plan.context_lens[i]) - int(plan.query_lens[i])
    q = state["q"][a + j0:a + j1]
    return (q, state["tables"][i:i + 1], np.array([c + j1], np.int32), np.array([0, j1 - j0], np.int32))


def oracle_timing_prefill(plan, seconds, rows_per_sample=None, state=None):
    """Time the multi-token oracle as it stands until ``seconds`` have
    passed (at least one sample): on whole sequences (all their new tokens,
    all heads), short ones first; or, with ``rows_per_sample``, on runs of
    that many consecutive new tokens of a sequence, each run computed as the
    request that ends at its last token (``prefill_row_request``; a run
    re-gathers its sequence's context, so runs cost more per FLOP than whole
    sequences).  With a
    ``state`` from ``oracle_state`` the samples continue where its previous
    sample stopped."""
    from oracle.prefill import paged_prefill_seqs

    st = state if state is not None else oracle_state(plan)
    scale = 1.0 / math.sqrt(plan.workload.head_size)
    order = [i for i in sorted(range(plan.B), key=lambda i: int(plan.context_lens[i]))  # short sequences first
             if int(plan.query_lens[i]) > 0]
    flops, seqs, rows = 0, 0, 0
    k, j0 = st["next"]
    t0 = time.perf_counter()
    while True:
        i = order[k % len(order)]
        n = int(plan.query_lens[i])
        if rows_per_sample is None:
            paged_prefill_seqs(st["q"], st["cache"], st["tables"], plan.context_lens, plan.query_start, scale, [i])
            flops += prefill_rows_flops(plan, i, 0, n)
            rows += n
            seqs += 1
            k += 1
        else:
            j1 = min(n, j0 + rows_per_sample)
            q, tables, cl, qs = prefill_row_request(plan, st, i, j0, j1)
            paged_prefill_seqs(q, st["cache"], tables, cl, qs, scale, [0])
            flops += prefill_rows_flops(plan, i, j0, j1)
            rows += j1 - j0
            j0 = j1
            if j0 >= n:
                k, j0 = k + 1, 0
                seqs += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    st["next"] = (k, j0)
    return {"tflops": flops / el / 1e12, "seconds": el, "seqs": seqs, "rows": rows, "cores": _threads()}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    plan = workload_plan(args.workload)
    state = oracle_state(plan)  # untimed: the oracle's copy of the workload
    # each step is a bounded sample, so that K steps take about ref_seconds
    per = min(5.0, args.ref_seconds / max(1, args.steps + args.warmup))
    if is_prefill(plan):
        for _ in range(args.warmup):
            oracle_timing_prefill(plan, per / 4, rows_per_sample=64, state=state)
        res = [oracle_timing_prefill(plan, per, rows_per_sample=64, state=state) for _ in range(max(1, args.steps))]
        tf = statistics.median(r["tflops"] for r in res)
        tot_s = sum(r["seconds"] for r in res)
        line = {
            "impl": "reference", "metric": PREFILL_METRIC, "value": round(tf, 6), "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000 * tot_s / max(1, args.steps), 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": {"workload": f"{plan.workload.name}: {plan.workload.description}",
                       "sample": "runs of 64 consecutive new tokens (all heads) of the step's sequences"},
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOP/s", "cores": res[0]["cores"], "kind": "oracle",
                             "sample": f"{sum(r['rows'] for r in res)} new tokens (all heads) in runs of 64, "
                                       f"about {per:.3f} s per step"},
            "e2e": {"value": round(tf, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    for _ in range(args.warmup):
        oracle_timing(plan, per / 4, max_rows=1, state=state)
    res = [oracle_timing(plan, per, state=state) for _ in range(max(1, args.steps))]
    gbs = statistics.median(r["gbs"] for r in res)
    tot_rows = sum(r["rows"] for r in res)
    tot_s = sum(r["seconds"] for r in res)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * tot_s / max(1, args.steps), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded lognormal lengths standing in for ShareGPT)",
        "config": {"workload": f"{plan.workload.name}: {plan.workload.description}", "sample": "whole rows"},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": res[0]["cores"], "kind": "oracle",
                         "sample": f"{tot_rows} sequences (all heads) of the workload, about {per:.3f} s per step"},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tok_per_s": round(tot_rows / tot_s, 3),
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())

    import paged_kv_cache_351_b200 as pa

    if args.tuning:
        pa.pa_set_decode_tuning(*[int(x) for x in args.tuning.split(",")])
    plan = workload_plan(args.workload, args.pool_gb)
    if is_prefill(plan):
        return run_prefill(args, plan, device, world, rank)
    w = plan.workload
    kv, inp = setup_device(plan, device)
    dev, tdt = inp["dev"], inp["tdt"]
    # shared-prefix decode when forks of one prompt share leading blocks
    groups = None
    gs_h, gb_h, max_group = kv.prefix_groups(plan.batch, w.num_heads)
    grouped = bool((gb_h > 0).any())
    if args.cascade == "on" or (args.cascade == "auto" and grouped):
        groups = (gs_h, gb_h, max_group)
    nbytes = step_bytes(plan, groups[:2] if groups else None)
    q = dev(inp["query"])
    key, value = dev(inp["key"]), dev(inp["value"])
    slots = torch.from_numpy(inp["slots"]).to(device)
    bt = torch.from_numpy(inp["tables"]).to(device)
    cl = torch.from_numpy(inp["lens"]).to(device)
    out = torch.empty_like(q)
    scale = 1.0 / math.sqrt(w.head_size)
    stream = torch.cuda.Stream(device)
    if groups:
        gs_d, gb_d = torch.from_numpy(groups[0]).to(device), torch.from_numpy(groups[1]).to(device)
        ws = kv.shared_workspace(plan.B, w.num_heads, groups[2], args.partition)
    else:
        ws = kv.workspace(plan.B, w.num_heads, bt.shape[1], args.partition)

    # cache write (when the step appends tokens) + decode (one launch, also
    # for a shared-prefix decode); fixed partitions add the merge kernel
    launches_per_step = (1 if len(inp["slots"]) else 0) + 1 + (1 if args.partition > 0 else 0)

    # the step as prepared library calls (descriptors built once), so that
    # per-step Python work does not leave the GPU idle between launches
    step = kv.prepare_step(slots, key, value, out, q, bt, cl, scale, partition_tokens=args.partition, stream=stream,
                           workspace=ws, groups=(gs_d, gb_d, groups[2]) if groups else None)

    K = args.steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    sampler = ClockSampler(uuid)
    time.sleep(0.25)
    # Warm-up right before the timed region (the sampler's start leaves the
    # GPU idle, and clocks drop when idle): W steps, continued until the GPU
    # has been busy for at least 50 ms.
    warm(step, stream, args.warmup)
    st, bits = pa.pa_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} bits {bits:#x} after warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # Timed region: K whole steps, events only at its ends (an event between
    # the write and the decode would block the decode's early launch).
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(K):
            step()
        ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed = ev0.elapsed_time(ev1)  # ms
    # Roofline of the dominant kernel: K decode launches on the same stream,
    # each bracketed by events, right after the timed region.
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    eb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with torch.cuda.stream(stream):
        for k in range(K):
            ea[k].record(stream)
            step.decode()
            eb[k].record(stream)
    torch.cuda.synchronize()
    dec_ms = statistics.mean(ea[k].elapsed_time(eb[k]) for k in range(K))
    # keep the same load a little longer if the timed region was too short for clock samples
    t_soak = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_soak < max(0.0, 0.6 - elapsed / 1000):
            for _ in range(50):
                step()
            torch.cuda.synchronize()
    clocks = sampler.stop()
    st, bits = pa.pa_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} bits {bits:#x} after the timed region")
    elapsed, dec_ms = max_over_ranks([elapsed, dec_ms], device, world)
    ms_step = elapsed / K
    value = aggregate_value(nbytes["step"], ms_step, world)
    tok_s = plan.B * world / (ms_step * 1e-3)
    peak, peak_kind = measured_peaks()

    # End to end through the public API: every step copies its inputs from
    # pinned host memory and reads its output back.  Two buffer sets let the
    # copies of steps k+1 (in) and k-1 (out) run on copy streams while step k
    # computes, as a serving loop would.
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e_decode(args, plan, kv, inp, out, scale, groups, nbytes, stream, device, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_timing(plan, args.cpu_seconds)
        cpu = {"value": round(r["gbs"], 4), "unit": "GB/s", "cores": r["cores"], "kind": "oracle",
               "sample": f"{r['rows']} whole sequences (all 32 heads) of the same workload in {r['seconds']:.1f} s"}

    achieved = nbytes["decode"] / (dec_ms * 1e-3) / 1e9
    traffic = ncu_traffic(profile_key(w.name, args.partition, groups is not None, grouped))
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; lognormal lengths stand in for ShareGPT)",
        "config": {"workload": f"{w.name}: {w.description}", "global_batch": plan.B * world,
                   "sum_context_tokens": int(sum(int(c) for c in plan.context_lens)),
                   "pool_blocks": plan.num_blocks, "partition_tokens": args.partition,
                   "parallelism": f"replicas x{world}",
                   "l2": f"no flush: the KV read per step ({nbytes['kv'] / 1e9:.2f} GB) exceeds the 126 MB L2"},
        "tok_per_s": round(tok_s, 1),
        "kv_read_gbs": round(nbytes["kv"] * world / (ms_step * 1e-3) / 1e9, 3),
        "shared_prefix": ({"groups": int(len(groups[1])), "groups_sharing": int((groups[1] > 0).sum()),
                           "max_group_size": groups[2], "kv_logical_bytes": nbytes["kv_logical"],
                           "kv_unique_bytes": nbytes["kv"],
                           "kv_logical_gbs": round(nbytes["kv_logical"] * world / (ms_step * 1e-3) / 1e9, 3),
                           "note": "value, kv_read_gbs and the roofline count each group's shared blocks once "
                                   "(the bytes the step must move); kv_logical_gbs counts them per member"}
                          if groups else None),
        "frac_of_hbm_peak": round(value / world / peak, 4),
        "frac_of_8tbs_spec": round(value / world / 8000.0, 4),
        "bytes_per_step": nbytes,
        "allocator": allocator_report(plan),
        "roofline": {"bound": "hbm",
                     "kernel": ("pa_decode_cascade (decode_kernel, shared-prefix groups, one launch)" if groups
                                else "pa_decode (decode_kernel + merge_fixed_kernel, fixed partitions)"
                                if args.partition > 0 else "pa_decode (decode_kernel, log-sum-exp merge fused)"),
                     "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": nbytes["decode"], "avg_launch_ms": round(dec_ms, 5),
                     "timing": f"{K} decode launches, each bracketed by CUDA events, after the timed region"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def pack_inputs(arrays, device):
    """One pinned host staging buffer holding the step's input arrays back
    to back (each at a 256-byte boundary), a device buffer of the same
    layout, and per array a function that views a buffer's segment as that
    array's dtype and shape."""
    import numpy as np
    import torch

    offs, off = [], 0
    for a in arrays:
        offs.append(off)
        off = (off + a.nbytes + 255) // 256 * 256
    host = torch.empty(max(off, 256), dtype=torch.uint8).pin_memory()
    hv = host.numpy()
    for a, o in zip(arrays, offs):
        hv[o:o + a.nbytes] = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    dev = torch.empty_like(host, device=device)
    tdt = {np.dtype(np.float32): torch.float32, np.dtype(np.uint16): torch.int16, np.dtype(np.int16): torch.int16,
           np.dtype(np.int32): torch.int32, np.dtype(np.int64): torch.int64}

    def viewer(a, o):
        return lambda buf: buf[o:o + a.nbytes].view(tdt[a.dtype]).view(a.shape)

    return host, dev, [viewer(a, o) for a, o in zip(arrays, offs)], off


def run_e2e_decode(args, plan, kv, inp, out, scale, groups, nbytes, stream, device, world):
    """End to end through the public API: each step copies its inputs from
    pinned host memory (one staging buffer: query, new K/V, slots, block
    tables, lengths and, for a shared-prefix decode, the groups) to the
    device, runs the step (cache write + decode, as prepared calls of the
    runtime helper) and copies the output back.  Two buffer sets let the
    copies of steps k+1 (in) and k-1 (out) run on copy streams while step k
    computes, as a serving loop would."""
    import numpy as np
    import torch
    import torch.distributed as dist

    w = plan.workload
    arrays = [inp["query"], inp["key"], inp["value"], inp["slots"], inp["tables"], inp["lens"]]
    if groups:
        arrays += [groups[0], groups[1]]
    bf = w.dtype == "bf16"
    view = (lambda t: t.view(torch.bfloat16)) if bf else (lambda t: t)
    sets = []
    for _ in range(2):
        host, dbuf, viewers, nbytes_in = pack_inputs(arrays, device)
        d = [f(dbuf) for f in viewers]
        d_out = torch.empty_like(out)
        grp = (d[6], d[7], groups[2]) if groups else None
        step = kv.prepare_step(d[3], view(d[1]), view(d[2]), d_out, view(d[0]), d[4], d[5], scale,
                               partition_tokens=args.partition, stream=stream, groups=grp)
        h_out = torch.empty(out.shape, dtype=torch.int16 if bf else torch.float32).pin_memory()
        sets.append({"host": host, "dev": dbuf, "out": d_out, "h_out": h_out, "step": step, "n_in": nbytes_in})
    h2d = sets[0]["n_in"]  # the packed staging buffer copied each step
    d2h = sets[0]["h_out"].numel() * sets[0]["h_out"].element_size()
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]

    def copy_in(k):
        b = k % 2
        if k >= 2:
            s_in.wait_event(ev_done[b])  # step k-2 no longer reads buffer set b
        with torch.cuda.stream(s_in):
            sets[b]["dev"].copy_(sets[b]["host"], non_blocking=True)
        ev_in[b].record(s_in)

    def compute(k):
        b = k % 2
        stream.wait_event(ev_in[b])
        if k >= 2:
            stream.wait_event(ev_read[b])  # step k-2's output has been read back
        sets[b]["step"]()
        ev_done[b].record(stream)

    def copy_out(k):
        b = k % 2
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            sets[b]["h_out"].copy_(sets[b]["out"].view(sets[b]["h_out"].dtype), non_blocking=True)
        ev_read[b].record(s_out)

    def run(n):
        copy_in(0)
        for k in range(n):
            if k + 1 < n:
                copy_in(k + 1)
            compute(k)
            copy_out(k)

    run(max(3, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    K = args.steps
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    stream.wait_event(f0)
    s_out.wait_event(f0)
    run(K)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    f1.record(s_out)
    torch.cuda.synchronize()
    e_ms = max_over_ranks([f0.elapsed_time(f1)], device, world)[0]
    e_step = e_ms / K
    iv = torch.int16 if bf else torch.int32
    if not torch.equal(sets[(K - 1) % 2]["h_out"].view(iv), out.view(iv).cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident step's output")
    return {"value": round(aggregate_value(nbytes["step"], e_step, world), 3), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(e_step, 5), "tok_per_s": round(plan.B * world / (e_step * 1e-3), 1),
            "overlap": "double-buffered: one packed copy in (step k+1) and one copy out (step k-1) overlap step k",
            "host_calls": "prepared library calls (descriptors built once per buffer set)"}


def run_prefill(args, plan, device, world, rank):
    """GPU arm for a multi-token (chunked-prefill) workload: a step writes
    the new tokens' K/V into the cache (pa_reshape_and_cache) and runs
    pa_prefill over them; value = the step's attention FLOPs / device time."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import paged_kv_cache_351_b200 as pa

    w = plan.workload
    flops = prefill_flops(plan)
    kv, inp = setup_device(plan, device)
    dev = inp["dev"]
    q, key, value = dev(inp["query"]), dev(inp["key"]), dev(inp["value"])
    slots = torch.from_numpy(inp["slots"]).to(device)
    bt = torch.from_numpy(inp["tables"]).to(device)
    cl = torch.from_numpy(inp["lens"]).to(device)
    qs = torch.from_numpy(plan.query_start).to(device)
    mq = int(plan.query_lens.max())
    out = torch.empty_like(q)
    scale = 1.0 / math.sqrt(w.head_size)
    stream = torch.cuda.Stream(device)
    T = plan.num_query_rows
    write_bytes = T * w.num_kv_heads * w.head_size * 2 * (w.elem_bytes + w.cache_elem_bytes) + 8 * T

    def attend(o, qq, b, c, s):
        pa.pa_prefill(o, qq, kv.k_cache, kv.v_cache, b, c, s, mq, scale, w.num_kv_heads, stream=stream)

    def step():
        kv.write(slots, key, value, None, stream=stream)
        attend(out, q, bt, cl, qs)

    K = args.steps
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    sampler = ClockSampler(uuid)
    time.sleep(0.25)
    warm(step, stream, args.warmup)
    st, bits = pa.pa_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} bits {bits:#x} after warm-up")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(K):
            step()
        ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed = ev0.elapsed_time(ev1)
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    eb = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    with torch.cuda.stream(stream):
        for k in range(K):
            ea[k].record(stream)
            attend(out, q, bt, cl, qs)
            eb[k].record(stream)
    torch.cuda.synchronize()
    pf_ms = statistics.mean(ea[k].elapsed_time(eb[k]) for k in range(K))
    t_soak = time.perf_counter()
    with torch.cuda.stream(stream):
        while time.perf_counter() - t_soak < max(0.0, 0.6 - elapsed / 1000):
            for _ in range(20):
                step()
            torch.cuda.synchronize()
    clocks = sampler.stop()
    st, bits = pa.pa_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} bits {bits:#x} after the timed region")
    elapsed, pf_ms = max_over_ranks([elapsed, pf_ms], device, world)
    ms_step = elapsed / K
    value = flops * world / (ms_step * 1e-3) / 1e12
    peak, peak_kind = measured_tensor_peak()

    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()  # noqa: E731
        h_in = (pin(inp["query"].view(np.int16)), pin(inp["key"].view(np.int16)), pin(inp["value"].view(np.int16)),
                pin(inp["slots"]), pin(inp["tables"]), pin(inp["lens"]), pin(plan.query_start))
        h_out = torch.empty(out.shape, dtype=torch.int16).pin_memory()
        d_in = tuple(torch.empty(x.shape, dtype=x.dtype, device=device) for x in h_in)
        h2d = sum(x.numel() * x.element_size() for x in h_in)
        d2h = h_out.numel() * h_out.element_size()
        bf = lambda t: t.view(torch.bfloat16)  # noqa: E731

        def e2e_step():
            for d, h in zip(d_in, h_in):
                d.copy_(h, non_blocking=True)
            d_q, d_k, d_v, d_s, d_bt, d_cl, d_qs = d_in
            kv.write(d_s, bf(d_k), bf(d_v), None, stream=stream)
            attend(out, bf(d_q), d_bt, d_cl, d_qs)
            h_out.copy_(out.view(torch.int16), non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(max(3, args.warmup)):
                e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            f0.record(stream)
            for _ in range(K):
                e2e_step()
            f1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks([f0.elapsed_time(f1)], device, world)[0] / K
        e2e = {"value": round(flops * world / (e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e_ms, 5),
               "overlap": "none: copies in, step, copy out, serialised on one stream"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = oracle_timing_prefill(plan, args.cpu_seconds)
        cpu = {"value": round(r["tflops"], 6), "unit": "TFLOP/s", "cores": r["cores"], "kind": "oracle",
               "sample": f"{r['seqs']} whole sequences (all new tokens, all heads) in {r['seconds']:.1f} s"}
    achieved = flops / (pf_ms * 1e-3) / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
        "config": {"workload": f"{w.name}: {w.description}", "query_rows": T, "sequences": plan.B,
                   "sum_context_tokens": int(plan.context_lens.sum()), "parallelism": f"replicas x{world}",
                   "l2": "no flush: each step rewrites the new tokens' K/V and reads "
                         f"{int(plan.context_lens.sum()) * 2 * w.num_kv_heads * w.head_size * 2 / 1e9:.2f} GB of "
                         "cache per kv head group; the kernel is tensor-bound"},
        "tokens_per_s": round(T * world / (ms_step * 1e-3), 1),
        "flops_per_step": flops, "write_bytes_per_step": write_bytes,
        "allocator": allocator_report(plan),
        "roofline": {"bound": "tensor", "kernel": "pa_prefill (prefill_kernel, tcgen05)", "achieved": round(achieved, 2),
                     "peak": peak, "peak_kind": peak_kind + " bf16 dense (burst)", "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": ncu_traffic(w.name, "prefill_kernel", PREFILL_SOURCES),
                     "traffic_unit": "DRAM bytes per launch", "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": round(pf_ms, 5),
                     "timing": f"{K} prefill launches, each bracketed by CUDA events, after the timed region"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
