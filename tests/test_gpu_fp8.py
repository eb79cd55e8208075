"""GPU parity of the FP8 (e4m3) KV cache against the oracle.

* pa_reshape_and_cache_fp8: the stored codes equal the oracle's
  e4m3(float(x) / scale[h]) bit for bit, from bf16 and from fp32 inputs,
  including values that saturate;
* pa_decode_fp8: max-abs error <= 1e-2 against the fp64 oracle computing on
  the dequantized codes (code value x scale), for edge lengths, group sizes
  and every split mode;
* the bf16-only entry points reject an FP8 cache.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import check_status_clean, to_device_values, to_host_raw
from oracle.attention import paged_decode, widen
from oracle.cache import PagedKVCache
from oracle.quant import quantize_kv
from workloads import to_bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128


def _scales(rng, hk):
    return (rng.uniform(0.5, 2.0, size=hk) * 5.0 / 448.0).astype(np.float32)


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
def test_fp8_write_bit_exact(in_dtype):
    rng = np.random.default_rng(5)
    T, hk, nb = 257, 4, 40
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[::13] = -1
    x = rng.standard_normal((T, hk, D)).astype(np.float32) * 2
    x[0, 0, :8] = [1e4, -1e4, 0.0, -0.0, 700.0 * 5 / 448, 1e-7, -1e-7, 3.0]
    y = rng.standard_normal((T, hk, D)).astype(np.float32)
    if in_dtype == "bf16":
        kx, vx = to_bf16_bits(x), to_bf16_bits(y)
        kf, vf = widen(kx, "bf16").astype(np.float32), widen(vx, "bf16").astype(np.float32)
    else:
        kx, vx, kf, vf = x, y, x, y
    ks, vs = _scales(rng, hk), _scales(rng, hk)
    kc = torch.zeros(nb, hk, 16, D, dtype=torch.float8_e4m3fn, device=DEV)
    vc = torch.zeros_like(kc)
    pa.pa_reshape_and_cache_fp8(to_device_values(kx, in_dtype, DEV), to_device_values(vx, in_dtype, DEV), kc, vc,
                                torch.from_numpy(slots).to(DEV), torch.from_numpy(ks).to(DEV),
                                torch.from_numpy(vs).to(DEV))
    check_status_clean()
    kq, vq = quantize_kv(kf, ks), quantize_kv(vf, vs)
    kh, vh = to_host_raw(kc, "fp8"), to_host_raw(vc, "fp8")
    for t, s in enumerate(slots.tolist()):
        if s < 0:
            continue
        assert np.array_equal(kh[s // 16, :, s % 16], kq[t]), t
        assert np.array_equal(vh[s // 16, :, s % 16], vq[t]), t


class Fp8Case:
    def __init__(self, seed, ctxs, H, hk, spare=5, q_mult=1.0):
        rng = np.random.default_rng(seed)
        self.ctxs, self.H, self.hk = list(ctxs), H, hk
        nbs = [-(-c // 16) for c in ctxs]
        self.NB = sum(nbs) + spare
        perm = rng.permutation(self.NB)
        self.max_nb = max(1, max(nbs)) + 2
        self.tables = np.full((len(ctxs), self.max_nb), -1, np.int32)
        slots, off = [], 0
        for i, (c, n) in enumerate(zip(ctxs, nbs)):
            self.tables[i, :n] = perm[off:off + n]
            off += n
            slots += [int(self.tables[i, t // 16]) * 16 + t % 16 for t in range(c)]
        T = len(slots)
        self.ks, self.vs = _scales(rng, hk), _scales(rng, hk)
        kx = to_bf16_bits(rng.standard_normal((T, hk, D)).astype(np.float32))
        vx = to_bf16_bits(rng.standard_normal((T, hk, D)).astype(np.float32))
        self.cache = PagedKVCache(self.NB, hk, D, 16, "fp8", self.ks, self.vs)
        self.cache.write(slots, quantize_kv(widen(kx, "bf16").astype(np.float32), self.ks),
                         quantize_kv(widen(vx, "bf16").astype(np.float32), self.vs))
        self.kc = torch.empty(self.NB, hk, 16, D, dtype=torch.float8_e4m3fn, device=DEV)
        self.kc.view(torch.uint8).fill_(0x7F)  # NaN codes in every slot never written
        self.vc = torch.empty_like(self.kc)
        self.vc.view(torch.uint8).fill_(0x7F)
        self.kst, self.vst = torch.from_numpy(self.ks).to(DEV), torch.from_numpy(self.vs).to(DEV)
        if T:
            pa.pa_reshape_and_cache_fp8(to_device_values(kx, "bf16", DEV), to_device_values(vx, "bf16", DEV),
                                        self.kc, self.vc, torch.tensor(slots, dtype=torch.int64, device=DEV),
                                        self.kst, self.vst)
        self.q = to_bf16_bits((rng.standard_normal((len(ctxs), H, D)) * q_mult).astype(np.float32))
        self.qd = to_device_values(self.q, "bf16", DEV)
        self.bt = torch.from_numpy(self.tables).to(DEV)
        self.cl = torch.tensor(ctxs, dtype=torch.int32, device=DEV)
        self.scale = 1.0 / math.sqrt(D)

    def run(self, mode):
        out = torch.empty_like(self.qd)
        n = pa.pa_decode_workspace_bytes(len(self.ctxs), self.H, self.hk, D, self.max_nb, mode)
        ws = torch.zeros(n + 256, dtype=torch.uint8, device=DEV) if n else None
        pa.pa_decode_fp8(out, self.qd, self.kc, self.vc, self.bt, self.cl, self.scale, self.hk, self.kst, self.vst,
                         workspace=ws, partition_tokens=mode)
        torch.cuda.synchronize()
        return out

    def err(self, out):
        ref = paged_decode(self.q, self.cache, self.tables, self.ctxs, self.scale)
        return float(np.max(np.abs(widen(to_host_raw(out, "bf16"), "bf16") - ref)))


EDGE_CTX = [0, 1, 15, 16, 17, 33, 100, 511, 512, 513, 1000, 2049]


@pytest.mark.parametrize("H,hk", [(8, 8), (16, 8), (32, 8), (16, 2)])
@pytest.mark.parametrize("mode", [0, -1, 64, 512])
def test_fp8_decode_parity(H, hk, mode):
    c = Fp8Case(60 + H + hk, EDGE_CTX, H, hk)
    out = c.run(mode)
    check_status_clean()
    assert not torch.isnan(out.float()).any()
    assert c.err(out) <= 1e-2


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values (8 significant bits) at |x| (normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("H,hk", [(8, 8), (16, 4), (16, 2)])
@pytest.mark.parametrize("q_mult", [1e-3, 3e3])
def test_fp8_decode_extreme_query_magnitudes(H, hk, q_mult):
    """The tensor-core page math carries the query as f16 high and low parts
    after scaling each head by a power of two; queries far larger (near
    one-hot softmax) or far smaller (near uniform) than N(0, 1) must still
    match the oracle at the plain bf16 bar: max-abs <= 1e-2 wherever
    |ref| < 4.  At |ref| >= 4 half a bf16 step is already 0.0156, so no
    bf16 output can promise 1e-2 there: those elements must be the correctly
    rounded bf16 value of the exact result, or its neighbour on the other
    side when the exact result lies within the fp32 computation's error
    (2^-12 relative) of a rounding midpoint; their error is printed in bf16
    steps."""
    c = Fp8Case(80 + H + hk, [1, 17, 100, 513, 2049], H, hk, q_mult=q_mult)
    ref = paged_decode(c.q, c.cache, c.tables, c.ctxs, c.scale)
    small = np.abs(ref) < 4.0
    ulp = bf16_ulp(ref)
    for mode in (0, -1):
        out = c.run(mode)
        got = widen(to_host_raw(out, "bf16"), "bf16")
        assert not np.isnan(got).any()
        err = np.abs(got - ref)
        err_small = float(err[small].max()) if small.any() else 0.0
        ulps = err[~small] / ulp[~small]
        # distance from ref to the nearest rounding midpoint, in bf16 steps
        frac = np.abs(ref[~small]) / ulp[~small]
        mid_dist = np.abs(frac - np.floor(frac) - 0.5)
        near_mid = mid_dist * ulp[~small] <= 2.0 ** -12 * np.abs(ref[~small])
        print(f"H={H} hk={hk} q_mult={q_mult} mode={mode}: max abs err {err_small:.3e} where |ref| < 4; "
              f"{int((~small).sum())} elements >= 4, max {float(ulps.max()) if ulps.size else 0.0:.3f} bf16 steps")
        assert err_small <= 1e-2, err_small
        assert np.all((ulps <= 0.5) | (near_mid & (ulps < 1.0))), ulps.max()
    check_status_clean()


def test_fp8_decode_random_batch():
    rng = np.random.default_rng(70)
    ctxs = rng.integers(0, 4000, size=150).tolist()
    c = Fp8Case(71, ctxs, 32, 8)
    for mode in (0, 512):
        assert c.err(c.run(mode)) <= 1e-2
    check_status_clean()


def test_bf16_entry_points_reject_fp8_cache():
    c = Fp8Case(72, [5], 4, 4)
    out = torch.empty_like(c.qd)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode(out, c.qd, c.kc, c.vc, c.bt, c.cl, c.scale, 4)
    assert e.value.status == 1
    key = torch.zeros(1, 4, D, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_reshape_and_cache(key, key, c.kc, c.vc, torch.zeros(1, dtype=torch.int64, device=DEV))
