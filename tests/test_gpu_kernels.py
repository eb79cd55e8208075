"""GPU parity of each kernel against the oracle, on small seeded cases that
still span several pages, partitions and workers, with ragged tails.

Bars: cache write and block copy bit-exact; decode max-abs error <= 1e-5
(fp32 KV) or <= 1e-2 (bf16 KV, output rounded to bf16) against the fp64
oracle.  The pool is filled with NaN before anything is written, so any
read of a slot the method never wrote would show up as NaN in the output.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import TOL, TORCH_DTYPE, check_status_clean, to_device_values, to_host_raw
from oracle.attention import attend_contiguous, paged_decode, partition_partials, widen
from oracle.cache import PagedKVCache
from workloads import to_bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _store(x, dtype):
    x = np.asarray(x, np.float32)
    return x if dtype == "f32" else to_bf16_bits(x)


def _nan_pool(nb, hk, d, dtype):
    t = torch.empty(nb, hk, 16, d, dtype=TORCH_DTYPE[dtype], device=DEV)
    t.fill_(float("nan"))
    return t


class Case:
    """Random K/V for each sequence scattered through a permuted block table,
    written on the GPU with pa_reshape_and_cache and into the oracle cache."""

    def __init__(self, seed, ctxs, H, Hkv, D, dtype, spare=7, pad_cols=3, q_stride_pad=0):
        rng = np.random.default_rng(seed)
        self.ctxs, self.H, self.Hkv, self.D, self.dtype = list(ctxs), H, Hkv, D, dtype
        nbs = [-(-c // 16) for c in ctxs]
        self.NB = sum(nbs) + spare
        perm = rng.permutation(self.NB)
        self.max_nb = max(1, max(nbs)) + pad_cols
        self.tables = np.full((len(ctxs), self.max_nb), -1, np.int32)
        off = 0
        slots_all, k_all, v_all = [], [], []
        for i, (c, n) in enumerate(zip(ctxs, nbs)):
            self.tables[i, :n] = perm[off:off + n]
            off += n
            slots_all += [int(self.tables[i, t // 16]) * 16 + t % 16 for t in range(c)]
            k_all.append(_store(rng.standard_normal((c, Hkv, D)), dtype))
            v_all.append(_store(rng.standard_normal((c, Hkv, D)), dtype))
        self.slots = np.asarray(slots_all, np.int64)
        self.k = np.concatenate(k_all) if k_all else np.zeros((0, Hkv, D))
        self.v = np.concatenate(v_all) if v_all else np.zeros((0, Hkv, D))
        self.cache = PagedKVCache(self.NB, Hkv, D, 16, dtype)
        self.cache.write(self.slots, self.k, self.v)
        self.kc = _nan_pool(self.NB, Hkv, D, dtype)
        self.vc = _nan_pool(self.NB, Hkv, D, dtype)
        if len(self.slots):
            pa.pa_reshape_and_cache(to_device_values(self.k, dtype, DEV), to_device_values(self.v, dtype, DEV),
                                    self.kc, self.vc, torch.from_numpy(self.slots).to(DEV))
        self.q = _store(rng.standard_normal((len(ctxs), H, D)), dtype)
        qd = to_device_values(self.q, dtype, DEV)
        if q_stride_pad:
            big = torch.zeros(len(ctxs), H + q_stride_pad, D, dtype=qd.dtype, device=DEV)
            big[:, :H] = qd
            qd = big[:, :H]
        self.qd = qd
        self.bt = torch.from_numpy(self.tables).to(DEV)
        self.cl = torch.from_numpy(np.asarray(ctxs, np.int32)).to(DEV)
        self.scale = 1.0 / math.sqrt(D)

    def oracle(self):
        return paged_decode(self.q, self.cache, self.tables, self.ctxs, self.scale)

    def run(self, partition_tokens=0, out=None, ws_extra=0):
        if out is None:
            out = torch.empty(len(self.ctxs), self.H, self.D, dtype=TORCH_DTYPE[self.dtype], device=DEV)
        n = pa.pa_decode_workspace_bytes(len(self.ctxs), self.H, self.Hkv, self.D, self.max_nb, partition_tokens)
        self.ws = torch.zeros(n + ws_extra + 256, dtype=torch.uint8, device=DEV) if n else None
        pa.pa_decode(out, self.qd, self.kc, self.vc, self.bt, self.cl, self.scale, self.Hkv, workspace=self.ws,
                     partition_tokens=partition_tokens)
        torch.cuda.synchronize()
        return out

    def err(self, out):
        got = widen(to_host_raw(out, self.dtype), self.dtype)
        return float(np.max(np.abs(got - self.oracle()))) if got.size else 0.0


EDGE_CTX = [0, 1, 15, 16, 17, 31, 33, 100, 511, 512, 513, 1000]


def test_wait_selftest_gives_up_and_context_survives():
    check_status_clean()
    pa.pa_debug_wait_selftest(timeout_ms=20)
    st, bits = pa.pa_get_device_status()
    assert st == 5 and bits & pa.PA_DEV_TIMEOUT
    check_status_clean()
    c = Case(1, [5, 40], 4, 4, 128, "bf16")
    assert c.err(c.run(-1)) <= TOL["bf16"]
    check_status_clean()


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 128)])
def test_reshape_and_cache_bit_exact(dtype, D):
    rng = np.random.default_rng(3)
    T, Hkv, NB = 300, 3, 40
    slots = rng.choice(NB * 16, size=T, replace=False).astype(np.int64)
    slots[::17] = -1
    k = _store(rng.standard_normal((T, Hkv, D)), dtype)
    v = _store(rng.standard_normal((T, Hkv, D)), dtype)
    kc, vc = _nan_pool(NB, Hkv, D, dtype), _nan_pool(NB, Hkv, D, dtype)
    # strided inputs: token stride padded, head stride padded
    kd = torch.zeros(T, Hkv + 1, D + 16, dtype=TORCH_DTYPE[dtype], device=DEV)
    kd[:, :Hkv, :D] = to_device_values(k, dtype, DEV)
    kview = kd[:, :Hkv, :D]
    pa.pa_reshape_and_cache(kview, to_device_values(v, dtype, DEV), kc, vc, torch.from_numpy(slots).to(DEV))
    check_status_clean()
    ref = PagedKVCache(NB, Hkv, D, 16, dtype)
    ref.write(slots, k, v)
    kh, vh = to_host_raw(kc, dtype), to_host_raw(vc, dtype)
    for b in ref.blocks():
        wr = ref.written(b)
        assert np.array_equal(kh[b][:, wr].view(np.uint32 if dtype == "f32" else np.uint16),
                              ref.k_page(b)[:, wr].view(np.uint32 if dtype == "f32" else np.uint16))
        assert np.array_equal(vh[b][:, wr].view(np.uint32 if dtype == "f32" else np.uint16),
                              ref.v_page(b)[:, wr].view(np.uint32 if dtype == "f32" else np.uint16))


def test_copy_blocks_bit_exact():
    rng = np.random.default_rng(4)
    NB, Hkv, D = 30, 5, 128
    kc = torch.randn(NB, Hkv, 16, D, device=DEV).to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, 16, D, device=DEV).to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    pairs = np.array([[3, 20], [7, 21], [3, 22], [29, 0]], np.int64)
    pa.pa_copy_blocks(kc, vc, torch.from_numpy(pairs).to(DEV))
    check_status_clean()
    ek, ev = k0.clone(), v0.clone()
    for s, d in pairs:
        ek[d] = k0[s]
        ev[d] = v0[s]
    assert torch.equal(kc.view(torch.int16), ek.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), ev.view(torch.int16))


def test_device_bounds_checks_flag_and_skip():
    check_status_clean()
    c = Case(5, [40, 20], 4, 2, 128, "bf16")
    # slot outside the pool: flagged, skipped, nothing else changes
    k0 = c.kc.clone()
    key = torch.zeros(2, 2, 128, dtype=torch.bfloat16, device=DEV)
    pa.pa_reshape_and_cache(key, key, c.kc, c.vc, torch.tensor([c.NB * 16, -5], dtype=torch.int64, device=DEV))
    st, bits = pa.pa_get_device_status()
    assert st == 6 and bits == pa.PA_DEV_BAD_SLOT
    assert torch.equal(c.kc.view(torch.int16), k0.view(torch.int16))
    # copy pair outside the pool
    pa.pa_copy_blocks(c.kc, c.vc, torch.tensor([[0, c.NB]], dtype=torch.int64, device=DEV))
    st, bits = pa.pa_get_device_status()
    assert st == 6 and bits == pa.PA_DEV_BAD_BLOCK
    # block-table entry outside the pool: flagged, page replaced by block 0
    bad = c.bt.clone()
    bad[0, 1] = c.NB + 100
    out = torch.empty_like(c.qd)
    pa.pa_decode(out, c.qd, c.kc, c.vc, bad, c.cl, c.scale, 2, partition_tokens=-1)
    st, bits = pa.pa_get_device_status()
    assert st == 6 and bits == pa.PA_DEV_BAD_BLOCK
    # context longer than the table row: flagged and clamped
    cl = c.cl.clone()
    cl[1] = c.max_nb * 16 + 5
    pa.pa_decode(out, c.qd, c.kc, c.vc, c.bt, cl, c.scale, 2, partition_tokens=-1)
    st, bits = pa.pa_get_device_status()
    assert st == 6 and bits & pa.PA_DEV_BAD_CONTEXT
    check_status_clean()


CONFIGS = [
    # dtype, D, H, Hkv
    ("f32", 64, 8, 8),
    ("bf16", 128, 32, 32),
    ("bf16", 128, 32, 8),
    ("bf16", 128, 16, 8),
    ("bf16", 128, 16, 2),
    ("bf16", 64, 8, 4),
    ("f32", 128, 4, 4),
    ("f32", 64, 8, 1),
]


@pytest.mark.parametrize("dtype,D,H,Hkv", CONFIGS)
@pytest.mark.parametrize("mode", [-1, 0, 16, 64, 512])
def test_decode_parity_edge_lengths(dtype, D, H, Hkv, mode):
    c = Case(11 + H + D, EDGE_CTX, H, Hkv, D, dtype)
    out = c.run(mode)
    check_status_clean()
    e = c.err(out)
    assert e <= TOL[dtype], f"max abs err {e}"
    assert not torch.isnan(out.float()).any()


@pytest.mark.parametrize("seed", range(3))
def test_decode_parity_random_batches(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 300))
    ctxs = rng.integers(0, 3000, size=B).tolist()
    c = Case(100 + seed, ctxs, 32, 8, 128, "bf16", q_stride_pad=8)
    for mode in (0, -1, 512):
        out = c.run(mode)
        check_status_clean()
        assert c.err(out) <= TOL["bf16"]


def test_output_strides():
    c = Case(21, [7, 300, 64], 8, 4, 128, "bf16")
    big = torch.zeros(3, 10, 128, dtype=torch.bfloat16, device=DEV)
    out = big[:, 1:9]
    c.run(0, out=out)
    assert c.err(out) <= TOL["bf16"]
    assert torch.all(big[:, 0] == 0) and torch.all(big[:, 9] == 0)


def test_fixed_partitions_leave_oracle_partials():
    """Fixed-partition mode leaves per-partition (o, lse) in the workspace;
    they match the oracle's per-partition restatement of the split step."""
    ctxs = [40, 700, 64, 1]
    part = 64
    c = Case(31, ctxs, 8, 4, 128, "bf16")
    c.run(part)
    B, H, D = len(ctxs), 8, 128
    P = -(-c.max_nb * 16 // part)
    nbytes_o = B * H * P * D * 4
    off_lse = (nbytes_o + 255) // 256 * 256
    ws = c.ws[pa.PA_DECODE_WS_HEADER_BYTES:]  # after the header of merge counters
    o = ws[:nbytes_o].view(torch.float32).view(B, H, P, D).cpu().numpy()
    lse = ws[off_lse:off_lse + B * H * P * 4].view(torch.float32).view(B, H, P).cpu().numpy()
    for i, ctx in enumerate(ctxs):
        npart = -(-ctx // part)
        if npart <= 1:
            continue
        from oracle.attention import gather_sequence

        k, v = gather_sequence(c.cache, c.tables[i], ctx)
        oo, ll = partition_partials(widen(c.q[i], "bf16"), k, v, c.scale, part)
        assert np.max(np.abs(o[i, :, :npart].transpose(1, 0, 2) - oo)) < 2e-5
        assert np.max(np.abs(lse[i, :, :npart].T - ll)) < 2e-5


def test_fixed_workspace_layout():
    """The fixed-partition workspace: the merge-counter header, o[B][H][P][D]
    and lse[B][H][P] (fp32, each rounded up to 256 bytes), then two share
    slots per worker for partitions cut between workers."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n = pa.pa_decode_workspace_bytes(8, 32, 8, 128, 8192, 512)
    P = 8192 * 16 // 512
    workers = sms * 16  # G = 4: 12 warps per SM over a bf16 cache, 16 over FP8 (the larger)
    shares = 2 * workers * 4 * 128 * 4 + (2 * workers * 4 * 4 + 255) // 256 * 256
    assert n == pa.PA_DECODE_WS_HEADER_BYTES + 8 * 32 * P * 128 * 4 + 8 * 32 * P * 4 + shares


def test_nosplit_is_bitwise_invariant_to_launch_shape():
    """Unsplit mode reduces each row in page order in one warp, so ring depth
    and warps per CTA must not change a single bit."""
    c = Case(41, [1, 100, 1000, 2049, 16, 17], 32, 8, 128, "bf16")
    ref = c.run(-1).clone()
    try:
        for warps, stages in ((8, 1), (8, 2), (4, 4), (2, 8), (1, 3)):
            pa.pa_set_decode_tuning(warps, stages, 1)
            assert torch.equal(c.run(-1).view(torch.int16), ref.view(torch.int16)), (warps, stages)
    finally:
        pa.pa_set_decode_tuning(0, 0, 0)


def test_balanced_split_under_other_launch_shapes():
    """The balanced split under other launch shapes, including grids of 4 and
    8 CTAs per SM that cannot all be resident at once (each CTA takes most of
    an SM's shared memory, so they run in waves): no worker waits for
    another, so every shape gives a correct result, the same bits on a second
    call, and leaves the workspace's merge counters at zero."""
    c = Case(42, [3000, 5, 900, 4096, 1], 32, 8, 128, "bf16")
    try:
        for warps, stages, ctas in ((8, 3, 1), (4, 2, 2), (1, 1, 1), (8, 1, 4), (12, 2, 8)):
            pa.pa_set_decode_tuning(warps, stages, ctas)
            first = c.run(0).clone()
            assert c.err(first) <= TOL["bf16"], (warps, stages, ctas)
            assert torch.equal(c.run(0).view(torch.int16), first.view(torch.int16)), (warps, stages, ctas)
            check_status_clean()
            assert int(c.ws[:pa.PA_DECODE_WS_HEADER_BYTES].count_nonzero()) == 0
    finally:
        pa.pa_set_decode_tuning(0, 0, 0)


def test_balanced_split_replays_from_a_cuda_graph():
    """A captured balanced-split decode replayed with new queries: each
    replay must equal a direct call on the same query (the merge counters
    are reset by the worker that completes each row, so a replay starts
    from zero like a fresh call)."""
    c = Case(45, [3000, 5, 900, 4096, 1, 700], 32, 8, 128, "bf16")
    n = pa.pa_decode_workspace_bytes(len(c.ctxs), c.H, c.Hkv, c.D, c.max_nb, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    q_static = c.qd.clone()
    out = torch.empty_like(q_static)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pa.pa_decode(out, q_static, c.kc, c.vc, c.bt, c.cl, c.scale, c.Hkv, workspace=ws, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        pa.pa_decode(out, q_static, c.kc, c.vc, c.bt, c.cl, c.scale, c.Hkv, workspace=ws, stream=s)
    gen = torch.Generator(device="cpu").manual_seed(3)
    for _ in range(3):
        q_new = torch.randn(q_static.shape, generator=gen).to(torch.bfloat16).to(DEV)
        q_static.copy_(q_new)
        g.replay()
        torch.cuda.synchronize()
        ref = torch.empty_like(out)
        ws2 = torch.zeros(n, dtype=torch.uint8, device=DEV)
        pa.pa_decode(ref, q_new, c.kc, c.vc, c.bt, c.cl, c.scale, c.Hkv, workspace=ws2)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    check_status_clean()
    assert int(ws[:pa.PA_DECODE_WS_HEADER_BYTES].count_nonzero()) == 0


def test_more_workers_than_pages():
    """Balanced mode with fewer pages than workers: empty workers sit inside
    rows that span several workers."""
    c = Case(43, [33, 17, 48], 4, 4, 128, "bf16")
    out = c.run(0)
    check_status_clean()
    assert c.err(out) <= TOL["bf16"]


def test_large_logit_range_is_stable():
    """Keys scaled x8 (like the outlier channels of the GQA workload, here on
    every channel) so logits span tens: the online softmax stays exact."""
    rng = np.random.default_rng(7)
    ctx = 600
    c = Case(44, [ctx], 4, 4, 128, "f32")
    k = (rng.standard_normal((ctx, 4, 128)) * 8).astype(np.float32)
    slots = torch.from_numpy(c.slots).to(DEV)
    pa.pa_reshape_and_cache(torch.from_numpy(k).to(DEV), torch.from_numpy(c.v).to(DEV), c.kc, c.vc, slots)
    c.cache.write(c.slots, k, c.v)
    for mode in (-1, 0, 128):
        assert c.err(c.run(mode)) <= TOL["f32"]
