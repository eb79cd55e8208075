"""GPU parity on the five seeded workloads at their full sizes, put on the
device through the library (C++ allocator -> pa_copy_blocks ->
pa_reshape_and_cache -> pa_decode) and checked against the oracle replay:

* block tables, slots and copy-on-write pairs: bit-exact (host allocator);
* cache contents of every block in use: bit-exact;
* decode outputs: max-abs error <= 1e-2 (bf16) / 1e-5 (fp32) on every row,
  or on a sampled set of rows for the largest workloads, in the launch
  configuration the benchmark times (auto mode) and in the fixed 512-token
  partition mode.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import (TOL, build_device_state, check_status_clean, decode_on_device, device_query,
                         max_abs_err, to_host_raw)
from oracle.attention import paged_decode_rows
from oracle.replay import block_table_array, replay
from workloads import make_plan, query_values

pytestmark = pytest.mark.gpu


def _check_cache(st, cache_o, blocks):
    w = st.plan.workload
    idx = torch.tensor(sorted(blocks), dtype=torch.int64, device="cuda")
    kc = st.k_cache.view(torch.uint8) if w.cache_dtype == "fp8" else st.k_cache
    vc = st.v_cache.view(torch.uint8) if w.cache_dtype == "fp8" else st.v_cache
    kh = to_host_raw(kc.index_select(0, idx), "fp8" if w.cache_dtype == "fp8" else w.dtype)
    vh = to_host_raw(vc.index_select(0, idx), "fp8" if w.cache_dtype == "fp8" else w.dtype)
    view = {"f32": np.uint32, "bf16": np.uint16, "fp8": np.uint8}[w.cache_dtype]
    for r, b in enumerate(sorted(blocks)):
        wr = cache_o.written(b)
        assert np.array_equal(kh[r][:, wr].view(view), cache_o.k_page(b)[:, wr].view(view)), b
        assert np.array_equal(vh[r][:, wr].view(view), cache_o.v_page(b)[:, wr].view(view)), b


def _run_workload(name, sample_rows=None, modes=(0, 512), check_all_blocks=True):
    plan = make_plan(name)
    st = build_device_state(plan, write_step=False)
    # the step: write the new tokens, then decode
    if st.step_slots is not None:
        st.write(st.step_key, st.step_value, st.step_slots)
    alloc_o, cache_o, log = replay(plan)
    assert np.array_equal(st.tables_host, block_table_array(alloc_o, plan.batch, plan.max_blocks_per_seq))
    assert np.array_equal(st.lens_host, plan.context_lens)
    assert st.cow_pairs == [p for _, _, c in log.appends for p in c]
    blocks = set(int(b) for b in st.tables_host.reshape(-1) if b >= 0)
    if not check_all_blocks:
        rng = np.random.default_rng(0)
        blocks = set(rng.choice(sorted(blocks), size=min(len(blocks), 4000), replace=False).tolist())
    _check_cache(st, cache_o, blocks)
    q = device_query(plan)
    rows = range(plan.B) if sample_rows is None else sample_rows
    ref = paged_decode_rows(query_values(plan), cache_o, st.tables_host, st.lens_host,
                            1.0 / math.sqrt(plan.workload.head_size), rows)
    errs = {}
    for mode in modes:
        out = decode_on_device(st, q, partition_tokens=mode)
        torch.cuda.synchronize()
        check_status_clean()
        errs[mode] = max_abs_err(out, ref, plan.workload.dtype)
        assert errs[mode] <= TOL[plan.workload.dtype], (mode, errs[mode])
    return st, errs


def test_tiny_fp32():
    _run_workload("tiny_fp32", modes=(0, -1, 16, 512))


def test_llama7b_bs64():
    _run_workload("llama7b_bs64", modes=(0, -1, 512))


def test_gqa_bs256():
    plan = make_plan("gqa_bs256")
    order = np.argsort(-plan.context_lens)
    rows = sorted(set(order[:6].tolist() + order[-4:].tolist() + list(range(0, 256, 16))))
    _run_workload("gqa_bs256", sample_rows=rows, modes=(0, 512), check_all_blocks=False)


def test_parallel_sampling_13b():
    st, _ = _run_workload("parallel_sampling_13b", modes=(0, -1))
    # 3 copies per prompt whose length is not a multiple of the block size
    plen = [op.n for op in st.plan.setup_ops if hasattr(op, "n") and op.n > 64]
    assert len(st.cow_pairs) == 3 * sum(1 for n in plen if n % 16)


def test_parallel_sampling_13b_shared_prefix():
    """The sampling workload through the shared-prefix decode: groups from
    the library's allocator (each prompt's 4 samples share its full
    blocks), every row against the oracle, in both split modes."""
    plan = make_plan("parallel_sampling_13b")
    st = build_device_state(plan)
    w = plan.workload
    gs, gb = st.alloc.prefix_groups(plan.batch, 4)
    assert len(gb) == 64 and list(np.diff(gs)) == [4] * 64 and (gb > 0).all()
    _, cache_o, _ = replay(plan)
    q = device_query(plan)
    ref = paged_decode_rows(query_values(plan), cache_o, st.tables_host, st.lens_host,
                            1.0 / math.sqrt(w.head_size), range(plan.B))
    gsd, gbd = torch.from_numpy(gs).cuda(), torch.from_numpy(gb).cuda()
    for mode in (0, -1):
        n = pa.pa_decode_cascade_workspace_bytes(plan.B, w.num_heads, w.num_kv_heads, w.head_size, 4, mode)
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
        out = torch.empty_like(q)
        pa.pa_decode_cascade(out, q, st.k_cache, st.v_cache, st.block_tables, st.context_lens, gsd, gbd, 4,
                             1.0 / math.sqrt(w.head_size), w.num_kv_heads, ws, partition_tokens=mode)
        torch.cuda.synchronize()
        check_status_clean()
        assert max_abs_err(out, ref, w.dtype) <= TOL[w.dtype], mode


def test_llama7b_bs64_fp8():
    _run_workload("llama7b_bs64_fp8", modes=(0, -1, 512))


def test_gqa_bs256_fp8():
    plan = make_plan("gqa_bs256_fp8")
    order = np.argsort(-plan.context_lens)
    rows = sorted(set(order[:6].tolist() + order[-4:].tolist() + list(range(0, 256, 16))))
    _run_workload("gqa_bs256_fp8", sample_rows=rows, modes=(0, 512), check_all_blocks=False)


def test_long_ctx_splitk():
    _run_workload("long_ctx_splitk", sample_rows=[0, 3, 7], modes=(512, 0), check_all_blocks=False)
