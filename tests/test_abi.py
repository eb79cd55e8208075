"""CPU-only checks of libpa.so: it loads, exports every function that
include/pa.h declares, rejects bad arguments before touching the GPU, and
its host allocator reproduces the oracle block manager bit for bit (slots,
copy-on-write pairs, tables, reference counts, free counts, waste) — on the
hand-worked example, on random request sequences and on the replays of
every seeded workload."""

import os
import random
import re

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from oracle.allocator import BlockAllocator, OutOfBlocks
from workloads import WORKLOADS, AddOp, AppendOp, ForkOp, make_plan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    with open(os.path.join(ROOT, "include", "pa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", text)))


def test_exports_every_declared_function():
    names = _declared_functions()
    assert len(names) >= 20
    lib = pa.library()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert lib.pa_version() == 1


def test_status_strings():
    lib = pa.library()
    for s in range(9):
        assert lib.pa_status_string(s) != b"unknown status"
    assert lib.pa_status_string(99) == b"unknown status"


def test_host_allocation_failure_is_a_status():
    """Host memory running out inside the allocator returns PA_ERR_HOST_ALLOC
    instead of letting a C++ exception cross the C ABI (which would end the
    process).  A child process caps its address space so that a pool of 2^30
    blocks cannot get its bookkeeping; a small pool in the same process keeps
    working."""
    import subprocess
    import sys

    code = (
        "import resource\n"
        "import paged_kv_cache_351_b200 as pa\n"
        "vm = [int(l.split()[1]) * 1024 for l in open('/proc/self/status') if l.startswith('VmSize:')][0]\n"
        "resource.setrlimit(resource.RLIMIT_AS, (vm + (1 << 30), resource.RLIM_INFINITY))\n"
        "small = pa.Allocator(1000, 16)\n"
        "try:\n"
        "    pa.Allocator(1 << 30, 16)\n"
        "except pa.PagedAttentionError as e:\n"
        "    print('status', e.status)\n"
        "small.add(0)\n"
        "small.append(0, 40)\n"
        "print('free', small.num_free())\n"
    )
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.split() == ["status", "8", "free", "997"]


# ---------------------------------------------------------------------------
# argument validation (returns before any CUDA call)
# ---------------------------------------------------------------------------

def _cache(nb=8, hk=2, d=128, dtype=torch.bfloat16):
    return torch.empty(nb, hk, 16, d, dtype=dtype)


def _expect(status, fn, *args, **kw):
    with pytest.raises(pa.PagedAttentionError) as e:
        fn(*args, **kw)
    assert e.value.status == status, str(e.value)


INVALID, UNSUPPORTED = 1, 2


def test_reshape_and_cache_validation():
    kc, vc = _cache(), _cache()
    key = torch.empty(4, 2, 128, dtype=torch.bfloat16)
    slots = torch.zeros(4, dtype=torch.int64)
    _expect(INVALID, pa.pa_reshape_and_cache, key, key, kc, vc, slots.to(torch.int32), stream=0)
    _expect(INVALID, pa.pa_reshape_and_cache, key[:3], key, kc, vc, slots, stream=0)
    _expect(INVALID, pa.pa_reshape_and_cache, key.float(), key.float(), kc, vc, slots, stream=0)
    _expect(INVALID, pa.pa_reshape_and_cache, key, key, kc, vc.float(), slots, stream=0)
    _expect(INVALID, pa.pa_reshape_and_cache, key, key, kc.transpose(0, 1), vc, slots, stream=0)
    _expect(UNSUPPORTED, pa.pa_reshape_and_cache, key[..., :96].contiguous(), key[..., :96].contiguous(),
            _cache(d=96), _cache(d=96), slots, stream=0)
    _expect(UNSUPPORTED, pa.pa_reshape_and_cache, key, key, torch.empty(8, 2, 32, 128, dtype=torch.bfloat16),
            torch.empty(8, 2, 32, 128, dtype=torch.bfloat16), slots, stream=0)
    # a token stride that is not a multiple of 16 bytes
    wide = torch.empty(4, 2, 132, dtype=torch.bfloat16)[..., :128]
    assert wide.stride(1) * 2 % 16 != 0
    _expect(INVALID, pa.pa_reshape_and_cache, wide, wide, kc, vc, slots, stream=0)


def test_copy_blocks_validation():
    kc, vc = _cache(), _cache()
    _expect(INVALID, pa.pa_copy_blocks, kc, vc, torch.zeros(3, 3, dtype=torch.int64), stream=0)
    _expect(INVALID, pa.pa_copy_blocks, kc, vc, torch.zeros(3, 2, dtype=torch.int32), stream=0)
    _expect(INVALID, pa.pa_copy_blocks, kc, vc, torch.zeros(2, 3, dtype=torch.int64).t(), stream=0)
    pa.pa_copy_blocks(kc, vc, torch.zeros(0, 2, dtype=torch.int64), stream=0)  # n == 0: nothing launched


def test_decode_validation():
    kc, vc = _cache(hk=2), _cache(hk=2)
    B, H = 3, 8
    q = torch.empty(B, H, 128, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    bt = torch.zeros(B, 4, dtype=torch.int32)
    cl = torch.zeros(B, dtype=torch.int32)
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt, cl, 0.1, 4, stream=0)  # num_kv_heads mismatch
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt.long(), cl, 0.1, 2, stream=0)
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt[:2], cl, 0.1, 2, stream=0)
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt, cl[:2], 0.1, 2, stream=0)
    _expect(INVALID, pa.pa_decode, out.float(), q, kc, vc, bt, cl, 0.1, 2, stream=0)
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt, cl, float("nan"), 2, stream=0)
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt.t().contiguous().t(), cl, 0.1, 2, stream=0)
    q6 = torch.empty(B, 6, 128, dtype=torch.bfloat16)
    _expect(UNSUPPORTED, pa.pa_decode, torch.empty_like(q6), q6, _cache(hk=2), _cache(hk=2), bt, cl, 0.1, 2,
            stream=0)  # group of 3
    q3 = torch.empty(B, 3, 128, dtype=torch.bfloat16)
    _expect(INVALID, pa.pa_decode, torch.empty_like(q3), q3, kc, vc, bt, cl, 0.1, 2, stream=0)  # H % H_kv
    # partition size not a multiple of the block size
    _expect(INVALID, pa.pa_decode, out, q, kc, vc, bt, cl, 0.1, 2, partition_tokens=100, stream=0)
    # B == 0: valid, nothing launched
    z = torch.empty(0, H, 128, dtype=torch.bfloat16)
    pa.pa_decode(z, z, kc, vc, torch.zeros(0, 4, dtype=torch.int32), torch.zeros(0, dtype=torch.int32), 0.1, 2,
                 stream=0)


def test_decode_cascade_validation():
    """Shared-prefix decode: argument errors are reported before any CUDA
    call (the group tensors, the group width, the split mode, the dtype)."""
    kc, vc = _cache(hk=2), _cache(hk=2)
    B, H = 4, 2
    q = torch.empty(B, H, 128, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    bt = torch.zeros(B, 4, dtype=torch.int32)
    cl = torch.zeros(B, dtype=torch.int32)
    gs = torch.tensor([0, 2, 4], dtype=torch.int32)
    gb = torch.tensor([1, 0], dtype=torch.int32)
    raw = torch.zeros((1 << 20) + 256, dtype=torch.uint8)
    ws = raw[(-raw.data_ptr()) % 256:][: 1 << 20]  # 256-byte aligned, as the workspace must be
    f = pa.pa_decode_cascade
    _expect(UNSUPPORTED, f, out, q, kc, vc, bt, cl, gs, gb, 3, 0.1, 2, ws, stream=0)  # G x 3 = 3 rows
    _expect(INVALID, f, out, q, kc, vc, bt, cl, gs, gb, 0, 0.1, 2, ws, stream=0)  # no member
    _expect(INVALID, f, out, q, kc, vc, bt, cl, gs[:2], gb, 2, 0.1, 2, ws, stream=0)  # [n_groups + 1]
    _expect(INVALID, f, out, q, kc, vc, bt, cl, gs.long(), gb, 2, 0.1, 2, ws, stream=0)
    _expect(INVALID, f, out, q, kc, vc, bt, cl, gs, gb[:0], 2, 0.1, 2, ws, stream=0)  # no group
    _expect(UNSUPPORTED, f, out, q, kc, vc, bt, cl, gs, gb, 2, 0.1, 2, ws, partition_tokens=512, stream=0)
    _expect(INVALID, f, out, q, kc, vc, bt, cl, gs, gb, 2, 0.1, 4, ws, stream=0)  # num_kv_heads mismatch
    k8, v8 = _cache(hk=2, dtype=torch.float8_e4m3fn), _cache(hk=2, dtype=torch.float8_e4m3fn)
    _expect(UNSUPPORTED, f, out, q, k8, v8, bt, cl, gs, gb, 2, 0.1, 2, ws, stream=0)
    q64 = torch.empty(B, H, 64, dtype=torch.bfloat16)
    _expect(UNSUPPORTED, f, torch.empty_like(q64), q64, _cache(hk=2, d=64), _cache(hk=2, d=64), bt, cl, gs, gb, 2,
            0.1, 2, ws, stream=0)  # bf16 at head size 64 has no shared-prefix kernels
    _expect(UNSUPPORTED, pa.pa_decode_cascade_workspace_bytes, B, H, 2, 128, 3)
    _expect(UNSUPPORTED, pa.pa_decode_cascade_workspace_bytes, B, H, 2, 128, 2, 512)
    _expect(INVALID, pa.pa_decode_cascade_workspace_bytes, B, H, 2, 128, 0)


def test_prefill_validation():
    kc, vc = _cache(hk=2), _cache(hk=2)
    B, T, H = 3, 10, 8
    q = torch.empty(T, H, 128, dtype=torch.bfloat16)
    out = torch.empty_like(q)
    bt = torch.zeros(B, 4, dtype=torch.int32)
    cl = torch.zeros(B, dtype=torch.int32)
    qs = torch.zeros(B + 1, dtype=torch.int32)
    f = pa.pa_prefill
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs, 4, 0.1, 4, stream=0)  # num_kv_heads mismatch
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs[:B], 4, 0.1, 2, stream=0)  # query_start not [B + 1]
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs.long(), 4, 0.1, 2, stream=0)
    _expect(INVALID, f, out, q, kc, vc, bt[:2], cl, qs, 4, 0.1, 2, stream=0)
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs, 4, 0.0, 2, stream=0)  # scale must be > 0
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs, 4, -0.1, 2, stream=0)
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs, 0, 0.1, 2, stream=0)  # T > 0 needs max_query_len > 0
    _expect(INVALID, f, out, q, kc, vc, bt, cl, qs, T + 1, 0.1, 2, stream=0)
    _expect(INVALID, f, out[:5], q, kc, vc, bt, cl, qs, 4, 0.1, 2, stream=0)
    _expect(UNSUPPORTED, f, out.float(), q.float(), _cache(hk=2, dtype=torch.float32),
            _cache(hk=2, dtype=torch.float32), bt, cl, qs, 4, 0.1, 2, stream=0)  # tensor-core path is bf16 only
    q64 = torch.empty(T, H, 64, dtype=torch.bfloat16)
    _expect(UNSUPPORTED, f, torch.empty_like(q64), q64, _cache(hk=2, d=64), _cache(hk=2, d=64), bt, cl, qs, 4, 0.1,
            2, stream=0)
    q6 = torch.empty(T, 6, 128, dtype=torch.bfloat16)
    _expect(UNSUPPORTED, f, torch.empty_like(q6), q6, kc, vc, bt, cl, qs, 4, 0.1, 2, stream=0)  # group of 3
    # nothing to compute: valid, nothing launched
    z = torch.empty(0, H, 128, dtype=torch.bfloat16)
    f(z, z, kc, vc, bt, cl, qs, 0, 0.1, 2, stream=0)
    f(out, q, kc, vc, torch.zeros(0, 4, dtype=torch.int32), torch.zeros(0, dtype=torch.int32),
      torch.zeros(1, dtype=torch.int32), 4, 0.1, 2, stream=0)


def test_empty_tensors_with_any_strides_are_accepted():
    """An empty batch is never read: the strides numpy gives empty arrays
    (all zero) must not be rejected, and nothing is launched."""
    empty = lambda *shape: torch.from_numpy(np.zeros(shape, np.uint16).view(np.int16)).view(torch.bfloat16)  # noqa: E731
    k = empty(0, 2, 128)
    assert k.stride() == (0, 0, 0)
    kc, vc = _cache(hk=2), _cache(hk=2)
    pa.pa_reshape_and_cache(k, k, kc, vc, torch.from_numpy(np.zeros(0, np.int64)), stream=0)
    q = empty(0, 4, 128)
    pa.pa_decode(q, q, kc, vc, torch.zeros(0, 4, dtype=torch.int32), torch.zeros(0, dtype=torch.int32), 0.1, 2,
                 stream=0)
    pa.pa_prefill(q, q, kc, vc, torch.zeros(2, 4, dtype=torch.int32), torch.zeros(2, dtype=torch.int32),
                  torch.zeros(3, dtype=torch.int32), 0, 0.1, 2, stream=0)


def test_device_of_a_call():
    """The binding makes the device holding a call's CUDA tensors current
    (the library launches on the current device); tensors on two devices are
    refused before anything runs, and host-only calls switch nothing."""
    from types import SimpleNamespace

    from paged_kv_cache_351_b200 import _device_index, _on_device

    on = lambda i: SimpleNamespace(device=torch.device("cuda", i))  # noqa: E731
    host = torch.empty(2)
    assert _device_index([host, None, np.zeros(2)]) is None
    assert _device_index([host, on(1), on(1), None]) == 1
    with pytest.raises(ValueError):
        _device_index([on(0), host, on(1)])
    with _on_device([host, None]):
        pass
    with pytest.raises(ValueError):
        _on_device([on(0), on(1)])


def test_workspace_size_without_a_device():
    """No split needs no workspace; the split modes size their share slots
    by the device's SM count, so without a device they report PA_ERR_CUDA
    (and bad arguments are still reported first)."""
    assert pa.PA_DECODE_WS_HEADER_BYTES == 64 * 1024
    assert pa.pa_decode_workspace_bytes(8, 32, 8, 128, 8192, -1) == 0
    _expect(INVALID, pa.pa_decode_workspace_bytes, 8, 32, 8, 128, 8192, 100)
    _expect(INVALID, pa.pa_decode_workspace_bytes, 8, 30, 8, 128, 8192, 0)
    if not torch.cuda.is_available():
        _expect(4, pa.pa_decode_workspace_bytes, 8, 32, 8, 128, 8192, 512)
        _expect(4, pa.pa_decode_workspace_bytes, 8, 32, 8, 128, 8192, 0)


# ---------------------------------------------------------------------------
# host allocator vs oracle
# ---------------------------------------------------------------------------

def _compare_state(c: pa.Allocator, o: BlockAllocator):
    assert c.num_free() == o.num_free()
    assert [c.refcount(b) for b in range(o.num_blocks)] == [o.refcount(b) for b in range(o.num_blocks)]
    for s in o.sequences():
        assert c.block_table(s) == o.block_table(s)
        assert c.length(s) == o.length(s)
    st = c.stats()
    assert st["num_free"] == o.num_free() and st["num_seqs"] == len(o.sequences())
    assert st["waste_slots"] == o.waste_slots()


@pytest.mark.parametrize("seed", range(8))
def test_allocator_matches_oracle_random(seed):
    rnd = random.Random(100 + seed)
    nb, bs = 40, 4
    order = list(range(nb))
    rnd.shuffle(order)
    c = pa.Allocator(nb, bs, order)
    o = BlockAllocator(nb, bs, order)
    live, nxt = [], 0
    for _ in range(400):
        r = rnd.random()
        if r < 0.12 or not live:
            c.add(nxt)
            o.add(nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.27:
            p = rnd.choice(live)
            c.fork(p, nxt)
            o.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.38:
            s = live.pop(rnd.randrange(len(live)))
            c.free(s)
            o.free(s)
        else:
            s = rnd.choice(live)
            n = rnd.choice([0, 1, 1, 2, 3, 4, 5, 9])
            try:
                oslots, ocow = o.append(s, n)
            except OutOfBlocks:
                with pytest.raises(pa.OutOfBlocksError):
                    c.append(s, n)
            else:
                cslots, ccow = c.append(s, n)
                assert cslots.tolist() == oslots and ccow == ocow
        _compare_state(c, o)


def test_allocator_golden_example():
    import json

    with open(os.path.join(ROOT, "tests", "golden", "fork_cow_example.json")) as f:
        g = json.load(f)
    c = pa.Allocator(g["num_blocks"], g["block_size"], g["free_order"])
    for stp in g["steps"]:
        if stp["op"] == "add":
            c.add(stp["seq"])
        elif stp["op"] == "fork":
            c.fork(stp["parent"], stp["child"])
        elif stp["op"] == "free":
            c.free(stp["seq"])
        elif stp.get("error"):
            with pytest.raises(pa.OutOfBlocksError):
                c.append(stp["seq"], stp["n"])
        else:
            slots, cow = c.append(stp["seq"], stp["n"])
            assert slots.tolist() == stp["slots"] and [list(p) for p in cow] == stp["cow"]
    fin = g["final"]
    assert [c.refcount(b) for b in range(g["num_blocks"])] == fin["refcounts"]
    assert c.stats()["waste_slots"] == fin["waste_slots"]
    for s, t in fin["tables"].items():
        assert c.block_table(int(s)) == t


def test_allocator_bad_requests():
    c = pa.Allocator(4, 4)
    c.add(1)
    for fn, args in ((c.add, (1,)), (c.append, (9, 1)), (c.fork, (9, 10)), (c.fork, (1, 1)), (c.free, (9,))):
        with pytest.raises(pa.PagedAttentionError):
            fn(*args)
    with pytest.raises(pa.PagedAttentionError):
        pa.Allocator(3, 4, [0, 1, 1])
    assert c.refcount(99) == -1


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_replay_matches_oracle(name):
    """Every seeded workload's request stream gives identical slots,
    copy-on-write pairs and block tables in C++ and in the oracle."""
    from oracle.replay import block_table_array, replay

    plan = make_plan(name)
    alloc_o, _, log = replay(plan, write_values=False)
    c = pa.Allocator(plan.num_blocks, plan.workload.block_size, plan.free_order)
    k = 0
    for op in plan.setup_ops + plan.step_ops:
        if isinstance(op, AddOp):
            c.add(op.seq)
        elif isinstance(op, ForkOp):
            c.fork(op.parent, op.child)
        elif isinstance(op, AppendOp):
            slots, cow = c.append(op.seq, op.n)
            seq, oslots, ocow = log.appends[k]
            k += 1
            assert seq == op.seq and np.array_equal(slots, np.asarray(oslots, np.int64)) and cow == ocow
    tables, lens = c.block_tables(plan.batch, plan.max_blocks_per_seq)
    assert np.array_equal(tables, block_table_array(alloc_o, plan.batch, plan.max_blocks_per_seq))
    assert np.array_equal(lens, plan.context_lens)
    assert c.stats()["waste_slots"] == alloc_o.waste_slots()


def test_append_batch_matches_single_appends():
    order = list(range(64))
    random.Random(3).shuffle(order)
    c1, c2 = pa.Allocator(64, 16, order), pa.Allocator(64, 16, order)
    for c in (c1, c2):
        for s in range(4):
            c.add(s)
            c.append(s, 10 + s)
        c.fork(0, 10)
        c.fork(1, 11)
    seqs, counts = [0, 10, 1, 11, 2, 3], [1, 1, 3, 1, 0, 20]
    slots_b, pairs_b = c1.append_batch(seqs, counts)
    slots_s, pairs_s = [], []
    for s, n in zip(seqs, counts):
        sl, cw = c2.append(s, n)
        slots_s += sl.tolist()
        pairs_s += cw
    assert slots_b.tolist() == slots_s and [tuple(p) for p in pairs_b.tolist()] == pairs_s


# ---------------------------------------------------------------------------
# prefix caching: C++ vs oracle
# ---------------------------------------------------------------------------

def test_prefix_cache_golden_example_cpp():
    from test_oracle_allocator import run_prefix_example

    a = run_prefix_example(pa.Allocator, lambda a, s, n: a.append(s, n), lambda a, s, t: a.append_tokens(s, t),
                           lambda a, s, t: a.add_prefix(s, t), lambda a: a.evictable(),
                           lambda a: a.stats()["num_cached"])
    assert a.num_free() == 0


@pytest.mark.parametrize("seed", range(8))
def test_prefix_cache_matches_oracle_random(seed):
    rnd = random.Random(300 + seed)
    nb, bs = 36, 4
    order = list(range(nb))
    rnd.shuffle(order)
    c = pa.Allocator(nb, bs, order)
    o = BlockAllocator(nb, bs, order)
    systems = [[rnd.randrange(3) for _ in range(rnd.choice([4, 8, 9, 12]))] for _ in range(3)]
    live, nxt, tracked = [], 0, set()
    for _ in range(500):
        r = rnd.random()
        if r < 0.25 or not live:
            prompt = rnd.choice(systems) + [rnd.randrange(3) for _ in range(rnd.randrange(0, 7))]
            hit_o = o.add_prefix(nxt, prompt)
            assert c.add_prefix(nxt, prompt) == hit_o
            live.append(nxt)
            tracked.add(nxt)
            toks = prompt[hit_o:]
            seq = nxt
            nxt += 1
            try:
                so, co = o.append_tokens(seq, toks)
            except OutOfBlocks:
                with pytest.raises(pa.OutOfBlocksError):
                    c.append_tokens(seq, toks)
            else:
                sc, cc = c.append_tokens(seq, toks)
                assert sc.tolist() == so and cc == co
        elif r < 0.35:
            p = rnd.choice(live)
            o.fork(p, nxt)
            c.fork(p, nxt)
            if p in tracked:
                tracked.add(nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.55:
            s = live.pop(rnd.randrange(len(live)))
            o.free(s)
            c.free(s)
            tracked.discard(s)
        else:
            s = rnd.choice(live)
            use_tokens = s in tracked and rnd.random() < 0.8
            if use_tokens:
                toks = [rnd.randrange(3) for _ in range(rnd.choice([1, 2, 3, 5]))]
                fo, fc = (lambda: o.append_tokens(s, toks)), (lambda: c.append_tokens(s, toks))
            else:
                tracked.discard(s)
                n = rnd.choice([1, 2, 5])
                fo, fc = (lambda: o.append(s, n)), (lambda: c.append(s, n))
            try:
                so, co = fo()
            except OutOfBlocks:
                with pytest.raises(pa.OutOfBlocksError):
                    fc()
            else:
                sc, cc = fc()
                assert sc.tolist() == so and cc == co
        _compare_state(c, o)
        assert c.evictable() == list(o._evictable)
        assert c.stats()["num_cached"] == o.num_cached()


def test_eviction_cascade_over_a_deep_branching_tree():
    """Evicting the root of a registered tree 500 blocks deep, with side
    branches at several depths, unregisters the descendants in the oracle's
    order (increasing block id, depth first) as the pool is drained a few
    blocks at a time."""
    import sys

    nb, bs, depth = 720, 4, 500
    rnd = random.Random(77)
    order = list(range(nb))
    rnd.shuffle(order)
    c, o = pa.Allocator(nb, bs, order), BlockAllocator(nb, bs, order)
    base = [rnd.randrange(5) for _ in range(depth * bs)]
    prompts = [base + [9]]
    for k in (50, 120, 121, 300, 499):
        prompts.append(base[: k * bs] + [5 + j % 3 for j in range(3 * bs)] + [9])
    limit = sys.getrecursionlimit()
    sys.setrecursionlimit(max(limit, 20 * depth))  # the oracle recurses once per tree level
    try:
        for s, prompt in enumerate(prompts):
            hit = o.add_prefix(s, prompt)
            assert c.add_prefix(s, prompt) == hit
            so, co = o.append_tokens(s, prompt[hit:])
            sc, cc = c.append_tokens(s, prompt[hit:])
            assert sc.tolist() == so and cc == co
        for s in (3, 0, 5, 1, 4, 2):
            o.free(s)
            c.free(s)
        assert c.evictable() == list(o._evictable) and len(c.evictable()) == depth + 5 * 3
        o.add(100)
        c.add(100)
        deepest = 0
        while o.num_free() > 0:
            n = min(37, o.num_free() * bs)
            before = o.num_cached()
            so, co = o.append(100, n)
            sc, cc = c.append(100, n)
            assert sc.tolist() == so and cc == co
            deepest = max(deepest, before - o.num_cached())
            _compare_state(c, o)
            assert c.evictable() == list(o._evictable)
            assert c.stats()["num_cached"] == o.num_cached()
        assert deepest > 100  # at least one request unregistered a subtree of over 100 blocks
    finally:
        sys.setrecursionlimit(limit)


def test_eviction_of_a_very_long_chain_keeps_the_host_stack():
    """A sequence of 100,000 registered blocks (1.6M tokens) freed and then
    evicted by one request: the cascade runs without recursion (a separate
    process, so a stack overflow would fail this test, not the test run)."""
    import subprocess
    import sys

    code = (
        "import numpy as np, paged_kv_cache_351_b200 as pa\n"
        "n, bs = 100000, 16\n"
        "a = pa.Allocator(n + 4, bs)\n"
        "toks = (np.arange(n * bs + 1) % 7 + 100 * (np.arange(n * bs + 1) // bs)).tolist()\n"
        "hit = a.add_prefix(0, toks)\n"
        "a.append_tokens(0, toks[hit:])\n"
        "a.free(0)\n"
        "assert len(a.evictable()) == n\n"
        "a.add(1)\n"
        "a.append(1, (n + 2) * bs)\n"
        "print('free', a.num_free(), 'evictable', len(a.evictable()))\n"
    )
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    assert res.stdout.split() == ["free", "2", "evictable", "0"]


@pytest.mark.parametrize("seed", range(6))
def test_swap_matches_oracle_random(seed):
    """Swap-out/in requests (with prefix caching and forks) give identical
    pairs, tables, host tables and free counts in C++ and in the oracle."""
    rnd = random.Random(500 + seed)
    nb, nh, bs = 24, 18, 4
    order = list(range(nb))
    rnd.shuffle(order)
    horder = list(range(nh))
    rnd.shuffle(horder)
    c, o = pa.Allocator(nb, bs, order), BlockAllocator(nb, bs, order)
    c.set_host_pool(nh, horder)
    o.set_host_pool(nh, horder)
    live, nxt = [], 0

    def both(fo, fc):
        try:
            ro = fo()
        except OutOfBlocks:
            with pytest.raises(pa.OutOfBlocksError):
                fc()
            return None
        rc = fc()
        return ro, rc

    for _ in range(500):
        resident = [s for s in live if not o.is_swapped(s)]
        swapped = [s for s in live if o.is_swapped(s)]
        r = rnd.random()
        if r < 0.2 or not live:
            prompt = [rnd.randrange(2) for _ in range(rnd.randrange(1, 14))]
            assert c.add_prefix(nxt, prompt) == o.add_prefix(nxt, prompt)
            hit = o.length(nxt)
            live.append(nxt)
            res = both(lambda: o.append_tokens(nxt, prompt[hit:]), lambda: c.append_tokens(nxt, prompt[hit:]))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
            nxt += 1
        elif r < 0.3 and resident:
            p = rnd.choice(resident)
            o.fork(p, nxt)
            c.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.45:
            s = live.pop(rnd.randrange(len(live)))
            o.free(s)
            c.free(s)
        elif r < 0.6 and resident:
            s = rnd.choice(resident)
            res = both(lambda: o.swap_out(s), lambda: c.swap_out(s))
            if res:
                assert [tuple(p) for p in res[1].tolist()] == res[0]
        elif r < 0.75 and swapped:
            s = rnd.choice(swapped)
            res = both(lambda: o.swap_in(s), lambda: c.swap_in(s))
            if res:
                assert [tuple(p) for p in res[1].tolist()] == res[0]
        elif resident:
            s = rnd.choice(resident)
            n = rnd.choice([1, 3])
            res = both(lambda: o.append(s, n), lambda: c.append(s, n))
            if res:
                assert res[1][0].tolist() == res[0][0] and res[1][1] == res[0][1]
        assert c.num_free() == o.num_free() and c.num_host_free() == o.num_host_free()
        for s in live:
            if o.is_swapped(s):
                assert c.host_table(s) == o.host_table(s)
            else:
                assert c.block_table(s) == o.block_table(s)
        assert c.evictable() == list(o._evictable)


def test_table_calls_report_the_size_they_need():
    """A table call given too little room fails with PA_ERR_INVALID_ARG,
    writes nothing, and reports the length it needs in *n_out."""
    import ctypes

    lib = pa.library()
    a = pa.Allocator(16, 4)
    a.add(3)
    a.append(3, 10)  # 3 blocks
    n = ctypes.c_int32(-1)
    out = (ctypes.c_int32 * 8)(*([-7] * 8))
    st = lib.pa_seq_block_table(a._h, 3, out, 2, ctypes.byref(n))
    assert st == 1 and n.value == 3 and list(out) == [-7] * 8
    st = lib.pa_seq_block_table(a._h, 3, out, n.value, ctypes.byref(n))
    assert st == 0 and list(out[:3]) == a.block_table(3) and out[3] == -7
