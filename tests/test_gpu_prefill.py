"""GPU parity of multi-token (chunked-prefill) paged attention (pa_prefill,
tensor cores) against the fp64 oracle.

* seeded workloads end to end: the cache is written through the allocator
  and pa_reshape_and_cache, then every new token attends causally; max-abs
  error <= 1e-2 (bf16) over every row (the small and the mixed
  chunk + decode workloads) or over sampled sequences (the 16 x 512 chunk
  workload, the launch the benchmark times);
* edge cases per group size G = 1, 2, 4, 8: empty sequences, single tokens,
  chunks spanning several 128-row tiles with ragged ends, contexts that are
  not a multiple of the block size, a pool whose unwritten slots hold NaN;
* rows outside every sequence stay untouched; a bad query_start is reported.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import build_device_state, check_status_clean, device_query, to_device_values, to_host_raw
from oracle.attention import widen
from oracle.cache import PagedKVCache
from oracle.prefill import paged_prefill, paged_prefill_seqs
from oracle.replay import block_table_array, replay
from workloads import make_plan, query_values, to_bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
D = 128
TOL = 1e-2


def _run_plan(plan, st, q):
    w = plan.workload
    out = torch.full_like(q, float("nan"))
    qs = torch.from_numpy(plan.query_start).to(DEV)
    pa.pa_prefill(out, q, st.k_cache, st.v_cache, st.block_tables, st.context_lens, qs,
                  int(plan.query_lens.max()), 1.0 / math.sqrt(w.head_size), w.num_kv_heads)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["prefill_tiny", "prefill_mixed_gqa"])
def test_prefill_workload_parity(name):
    plan = make_plan(name)
    st = build_device_state(plan)
    alloc_o, cache_o, _ = replay(plan)
    assert np.array_equal(st.tables_host, block_table_array(alloc_o, plan.batch, plan.max_blocks_per_seq))
    out = _run_plan(plan, st, device_query(plan))
    check_status_clean()
    ref = paged_prefill(query_values(plan), cache_o, st.tables_host, plan.context_lens, plan.query_start,
                        1.0 / math.sqrt(D))
    got = widen(to_host_raw(out, "bf16"), "bf16")
    assert float(np.max(np.abs(got - ref))) <= TOL


def test_prefill_chunks_llama7b_sampled():
    """The 16 x 512-token chunk workload at full size, in the launch the
    benchmark times; the oracle recomputes three whole sequences."""
    plan = make_plan("prefill_chunks_llama7b")
    st = build_device_state(plan)
    out = _run_plan(plan, st, device_query(plan))
    check_status_clean()
    _, cache_o, _ = replay(plan)
    seqs = [int(np.argmax(plan.context_lens)), int(np.argmin(plan.context_lens)), 5]
    rows = paged_prefill_seqs(query_values(plan), cache_o, st.tables_host, plan.context_lens, plan.query_start,
                              1.0 / math.sqrt(D), seqs)
    got = widen(to_host_raw(out, "bf16"), "bf16")
    for i in seqs:
        a, e = int(plan.query_start[i]), int(plan.query_start[i + 1])
        assert float(np.max(np.abs(got[a:e] - rows[i]))) <= TOL, i
    assert not torch.isnan(out.float()).any()


class Case:
    """(prior, new) pairs over permuted blocks of a NaN-filled pool."""

    def __init__(self, seed, pairs, H, hk, extra_rows=0):
        rng = np.random.default_rng(seed)
        self.pairs, self.H, self.hk = pairs, H, hk
        self.ctx = np.array([a + b for a, b in pairs], np.int32)
        self.qlen = np.array([b for _, b in pairs], np.int32)
        self.qs = np.concatenate([[0], np.cumsum(self.qlen)]).astype(np.int32)
        self.T = int(self.qs[-1]) + extra_rows
        nbs = [-(-int(c) // 16) for c in self.ctx]
        self.NB = sum(nbs) + 4
        perm = rng.permutation(self.NB)
        self.max_nb = max(1, max(nbs)) + 1
        self.tables = np.full((len(pairs), self.max_nb), -1, np.int32)
        slots, off = [], 0
        for i, (c, n) in enumerate(zip(self.ctx.tolist(), nbs)):
            self.tables[i, :n] = perm[off:off + n]
            off += n
            slots += [int(self.tables[i, t // 16]) * 16 + t % 16 for t in range(c)]
        k = to_bf16_bits(rng.standard_normal((len(slots), hk, D)).astype(np.float32))
        v = to_bf16_bits(rng.standard_normal((len(slots), hk, D)).astype(np.float32))
        self.cache = PagedKVCache(self.NB, hk, D, 16, "bf16")
        self.cache.write(slots, k, v)
        self.kc = torch.full((self.NB, hk, 16, D), float("nan"), dtype=torch.bfloat16, device=DEV)
        self.vc = torch.full_like(self.kc, float("nan"))
        if slots:
            pa.pa_reshape_and_cache(to_device_values(k, "bf16", DEV), to_device_values(v, "bf16", DEV), self.kc,
                                    self.vc, torch.tensor(slots, dtype=torch.int64, device=DEV))
        self.q = to_bf16_bits(rng.standard_normal((self.T, H, D)).astype(np.float32))
        self.scale = 1.0 / math.sqrt(D)

    def run(self, max_q=None, qs=None):
        out = torch.full((self.T, self.H, D), 7.0, dtype=torch.bfloat16, device=DEV)
        pa.pa_prefill(out, to_device_values(self.q, "bf16", DEV), self.kc, self.vc,
                      torch.from_numpy(self.tables).to(DEV), torch.from_numpy(self.ctx).to(DEV),
                      torch.from_numpy(self.qs if qs is None else qs).to(DEV),
                      int(max(1, self.qlen.max())) if max_q is None else max_q, self.scale, self.hk)
        torch.cuda.synchronize()
        return out

    def ref(self):
        return paged_prefill(self.q[: int(self.qs[-1])], self.cache, self.tables, self.ctx, self.qs, self.scale)


EDGE = [(0, 1), (0, 17), (23, 7), (0, 300), (16, 16), (100, 129), (511, 1), (257, 256), (40, 0), (0, 0), (5, 33),
        (1000, 200), (127, 1), (128, 128), (3, 250)]


@pytest.mark.parametrize("H,hk", [(8, 8), (16, 8), (16, 4), (16, 2)])
def test_prefill_edge_cases(H, hk):
    c = Case(40 + H + hk, EDGE, H, hk, extra_rows=3)
    out = c.run()
    check_status_clean()
    got = widen(to_host_raw(out, "bf16"), "bf16")
    n = int(c.qs[-1])
    assert not np.isnan(got[:n]).any()
    assert float(np.max(np.abs(got[:n] - c.ref()))) <= TOL
    assert np.all(got[n:] == 7.0)  # rows outside every sequence are not written


def test_prefill_single_tokens_match_decode():
    """n_i = 1 rows are decode rows: pa_prefill and pa_decode agree with the
    oracle on the same cache."""
    ctxs = [1, 2, 15, 16, 17, 200, 513, 1500]
    c = Case(50, [(x - 1, 1) for x in ctxs], 32, 8)
    out_p = c.run()
    out_d = torch.empty_like(out_p)
    q = to_device_values(c.q, "bf16", DEV)
    pa.pa_decode(out_d, q, c.kc, c.vc, torch.from_numpy(c.tables).to(DEV), torch.from_numpy(c.ctx).to(DEV),
                 c.scale, c.hk, partition_tokens=-1)
    check_status_clean()
    ref = c.ref()
    for out in (out_p, out_d):
        assert float(np.max(np.abs(widen(to_host_raw(out, "bf16"), "bf16") - ref))) <= TOL


def test_prefill_reports_bad_query_start():
    c = Case(51, [(10, 5), (0, 4)], 8, 8)
    bad = c.qs.copy()
    bad[1] = 40  # more new tokens than the sequence's context
    c.run(qs=bad)
    st, bits = pa.pa_get_device_status()
    assert bits & 0x4
    c2 = Case(52, [(10, 600)], 8, 8)
    c2.run(max_q=5)  # max_query_len so small that the grid misses rows of a sequence
    st, bits = pa.pa_get_device_status()
    assert bits & 0x4
    check_status_clean()
