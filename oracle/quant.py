"""FP8 (e4m3) KV-cache codes — oracle (test infrastructure; see the package
header).

The pages say only that the KV cache itself can be quantized to save memory
(gitcode repo walkthrough, section 三 "量化", the quantized_kvcache item).
The reading taken here: each stored K (or V) value is an OCP FP8 e4m3 code of
the value divided by a per-kv-head scale,

    code = e4m3(float32(x) / float32(scale[h]))      (IEEE fp32 division)
    value = e4m3_value(code) * scale[h]

with e4m3 = 1 sign, 4 exponent (bias 7), 3 mantissa bits, no infinities,
0x7F/0xFF = NaN, largest finite 448; rounding to nearest with ties to the
even code; finite values beyond the range saturate to +-448.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """Exact value of each code (fp64); NaN for 0x7F and 0xFF."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


# magnitudes of the finite non-negative codes 0x00..0x7E, increasing
_MAGS = e4m3_decode(np.arange(0x7F, dtype=np.uint8))


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round float32 values to e4m3 codes: nearest, ties to the even code,
    finite values beyond +-448 (and infinities) saturate, NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    hi = np.clip(np.searchsorted(_MAGS, a, side="left"), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = np.abs(_MAGS[hi] - a)
    d_lo = np.abs(a - _MAGS[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(a >= E4M3_MAX, 0x7E, code)  # saturate (includes +-inf)
    code = code.astype(np.uint8) | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


def quantize_kv(x_f32: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x [T, H_kv, D] float32 (the exact widening of the inputs), scale
    [H_kv] float32 -> codes [T, H_kv, D] uint8."""
    x = np.asarray(x_f32, dtype=np.float32)
    s = np.asarray(scale, dtype=np.float32)[None, :, None]
    return e4m3_encode((x / s).astype(np.float32))
