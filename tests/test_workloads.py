"""The seeded generators: reproducible, shaped as documented, and the bf16
rounding agrees with torch's round-to-nearest-even conversion."""

import numpy as np
import torch

from workloads import (WORKLOADS, AppendOp, bf16_bits_to_f32, make_plan, query_values,
                       stream_kv, to_bf16_bits)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -2.5], np.float32)])
    ours = to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_plans_are_reproducible_and_shaped():
    for name, w in WORKLOADS.items():
        p1, p2 = make_plan(name), make_plan(name)
        assert np.array_equal(p1.context_lens, p2.context_lens)
        assert np.array_equal(p1.free_order, p2.free_order)
        assert sorted(p1.free_order.tolist()) == list(range(p1.num_blocks))
        assert p1.context_lens.shape[0] == p1.B
        q = query_values(p1)
        rows = p1.B if np.all(p1.query_lens == 1) else p1.num_query_rows
        assert q.shape == (rows, w.num_heads, w.head_size)
        assert p1.query_start[-1] == p1.num_query_rows and np.all(p1.query_lens <= p1.context_lens)


def test_documented_sizes():
    p = make_plan("tiny_fp32")
    assert p.context_lens.tolist() == [1, 17, 33, 100] and p.num_blocks == 64
    p = make_plan("llama7b_bs64")
    assert p.B == 64 and p.num_blocks == 152587
    assert p.context_lens.min() >= 16 and p.context_lens.max() <= 2048
    assert 25_000 < int(p.context_lens.sum()) < 70_000
    p = make_plan("gqa_bs256")
    assert p.B == 256 and p.outlier_channels.shape == (10, 2)
    assert p.context_lens.min() >= 32 and p.context_lens.max() <= 8192
    p = make_plan("long_ctx_splitk")
    assert int(p.context_lens.sum()) == 704512
    p = make_plan("parallel_sampling_13b")
    assert p.B == 256 and p.context_lens.max() <= 1024 + 64
    p = make_plan("prefill_chunks_llama7b")
    assert p.B == 16 and p.num_query_rows == 16 * 512 and p.context_lens.max() <= 3584 + 512
    p = make_plan("prefill_mixed_gqa")
    assert p.B == 64 and p.num_query_rows == 4 * 512 + 60
    assert p.query_lens.tolist() == [512] * 4 + [1] * 60
    p = make_plan("prefill_tiny")
    assert (0 in p.query_lens.tolist()) and (0 in p.context_lens.tolist())


def test_prefill_step_appends_new_tokens_after_prior_context():
    for name in ("prefill_tiny", "prefill_mixed_gqa"):
        p = make_plan(name)
        step = {op.seq: op for op in p.step_ops}
        for i in range(p.B):
            q, c = int(p.query_lens[i]), int(p.context_lens[i])
            if q == 0:
                assert i not in step
            else:
                assert step[i].n == q and step[i].start == c - q and step[i].stream == i


def test_stream_slices_agree_across_chunks():
    p = make_plan("gqa_bs256")
    k_all, v_all = stream_kv(p, 3, 0, 2500)
    for a, n in ((1000, 100), (0, 1), (1023, 2), (2047, 453), (5, 17)):
        k_mid, v_mid = stream_kv(p, 3, a, n)
        assert np.array_equal(k_all[a:a + n], k_mid) and np.array_equal(v_all[a:a + n], v_mid)
    # outlier channels are scaled in K only
    kf = bf16_bits_to_f32(k_all)
    h, d = p.outlier_channels[0]
    assert np.abs(kf[:, h, d]).mean() > 4 * np.abs(kf[:, (h + 1) % 8, d]).mean()


def test_step_appends_last_position():
    p = make_plan("llama7b_bs64")
    assert len(p.step_ops) == 64
    for i, op in enumerate(p.step_ops):
        assert isinstance(op, AppendOp) and op.n == 1 and op.start == p.context_lens[i] - 1
