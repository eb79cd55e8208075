"""Pins for the oracle's FP8 (e4m3) KV codes.

* decoding every one of the 256 codes agrees with torch's float8_e4m3fn;
* encoding agrees with torch's (round-to-nearest-even) conversion for every
  value torch maps to a finite code, including subnormals and exact ties;
* every finite code round-trips; the largest finite value is 448;
* saturation (the reading for values beyond the range): finite values at or
  above the rounding threshold and infinities give +-448, NaN gives 0x7F;
* the per-head quantization divides in fp32 and keeps the sign of zero;
* planted mistakes (ties away from zero, wrong exponent bias) are caught.
"""

import numpy as np
import pytest
import torch

from oracle import quant
from oracle.attention import gather_sequence, widen
from oracle.replay import replay
from workloads import kv_scales, make_plan, seq_token_sources, stream_kv


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def _torch_encode(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_decode_all_codes_match_torch():
    c = np.arange(256, dtype=np.uint8)
    ours, ref = quant.e4m3_decode(c), _torch_decode(c)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert quant.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert quant.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9


def _encode_pin(encode):
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 40,
        rng.standard_normal(20000).astype(np.float32) * 0.01,
        # exact midpoints between neighbouring codes (ties), both signs
        ((quant.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8)) +
          quant.e4m3_decode(np.arange(1, 0x7F, dtype=np.uint8))) / 2).astype(np.float32),
        -((quant.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8)) +
           quant.e4m3_decode(np.arange(1, 0x7F, dtype=np.uint8))) / 2).astype(np.float32),
        np.array([0.0, -0.0, 448.0, -448.0, 460.0, 2.0 ** -10, 1.5 * 2.0 ** -9], np.float32),
    ])
    x = x[np.abs(x) < 464.0]  # beyond this torch gives NaN where the reading saturates
    assert np.array_equal(encode(x), _torch_encode(x))


def test_encode_matches_torch():
    _encode_pin(quant.e4m3_encode)


def test_round_trip_and_saturation():
    c = np.array([k for k in range(256) if k not in (0x7F, 0xFF)], np.uint8)
    assert np.array_equal(quant.e4m3_encode(quant.e4m3_decode(c).astype(np.float32)), c)
    big = np.array([464.0, 480.0, 1e6, np.inf, -464.0, -1e30, -np.inf], np.float32)
    assert quant.e4m3_encode(big).tolist() == [0x7E] * 4 + [0xFE] * 3
    assert quant.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_quantize_kv_divides_per_head_in_fp32():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 3, 8)).astype(np.float32)
    x[0, 0, 0] = -0.0
    s = np.array([0.0133, 0.5, 3.0], np.float32)
    codes = quant.quantize_kv(x, s)
    for t in range(50):
        for h in range(3):
            y = np.array([np.float32(v) / np.float32(s[h]) for v in x[t, h]], np.float32)
            assert np.array_equal(codes[t, h], _torch_encode(y))
    assert codes[0, 0, 0] == 0x80


class _TiesAway:
    @staticmethod
    def encode(x):
        c = quant.e4m3_encode(x)
        a = np.abs(x.astype(np.float64))
        lo = quant.e4m3_decode(c & 0x7F)
        nxt = quant.e4m3_decode(np.minimum((c & 0x7F) + 1, 0x7E).astype(np.uint8))
        tie = (nxt - a) == (a - lo)
        return np.where(tie & (a < 448), c + 1, c).astype(np.uint8)


def _wrong_bias(x):
    return quant.e4m3_encode(np.asarray(x, np.float32) * np.float32(2.0))


@pytest.mark.parametrize("mutant", [_TiesAway.encode, _wrong_bias])
def test_pins_catch_planted_mistakes(mutant):
    with pytest.raises(AssertionError):
        _encode_pin(mutant)


def test_fp8_replay_reads_back_quantized_history():
    plan = make_plan("gqa_bs256_fp8")
    plan.setup_ops = [op for op in plan.setup_ops if getattr(op, "seq", 0) < 3]
    plan.step_ops = [op for op in plan.step_ops if op.seq < 3]
    alloc, cache, _ = replay(plan)
    ks, vs = kv_scales(plan)
    runs = seq_token_sources(plan)
    for sid in range(3):
        k_parts, v_parts = zip(*[stream_kv(plan, st, a, n) for st, a, n in runs[sid]])
        k = widen(np.concatenate(k_parts), "bf16").astype(np.float32)
        v = widen(np.concatenate(v_parts), "bf16").astype(np.float32)
        k_ref = quant.e4m3_decode(quant.quantize_kv(k, ks)) * ks.astype(np.float64)[None, :, None]
        v_ref = quant.e4m3_decode(quant.quantize_kv(v, vs)) * vs.astype(np.float64)[None, :, None]
        kg, vg = gather_sequence(cache, alloc.block_table(sid), alloc.length(sid))
        assert np.array_equal(kg, k_ref) and np.array_equal(vg, v_ref)
        # quantization error is bounded by half a code step times the scale
        assert np.max(np.abs(kg - k) / ks[None, :, None]) <= 16.0 + 1e-9
