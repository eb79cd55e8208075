"""Block swapping end to end on the GPU: sequences are swapped out to a
pinned host pool (allocator pairs + pa_swap_blocks), their device blocks are
reused and overwritten by new sequences, then they are swapped back in and
decoded.  The cache bytes of every live block equal the oracle's (which
applies the same pairs between its own device and host pools), and every
decode output matches the oracle (max-abs <= 1e-2, bf16).  Pageable host
memory is refused before any launch."""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import check_status_clean, to_device_values, to_host_raw
from oracle.allocator import BlockAllocator
from oracle.attention import paged_decode, widen
from oracle.cache import PagedKVCache
from oracle.replay import block_table_array
from workloads import to_bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
HK, H, D, BS = 4, 8, 128, 16


def test_swap_out_reuse_swap_in_decode():
    rng = np.random.default_rng(21)
    NB, NH = 120, 60
    order = rng.permutation(NB).astype(np.int32)
    horder = rng.permutation(NH).astype(np.int32)
    c, o = pa.Allocator(NB, BS, order), BlockAllocator(NB, BS, order)
    c.set_host_pool(NH, horder)
    o.set_host_pool(NH, horder)
    dev_o = PagedKVCache(NB, HK, D, BS, "bf16")
    host_o = PagedKVCache(NH, HK, D, BS, "bf16")
    kc = torch.empty(NB, HK, BS, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.empty_like(kc)
    kh = torch.empty(NH, HK, BS, D, dtype=torch.bfloat16).pin_memory()
    vh = torch.empty_like(kh).pin_memory()

    def add(s, n):
        c.add(s)
        o.add(s)
        slots, _ = c.append(s, n)
        so, _ = o.append(s, n)
        assert slots.tolist() == so
        k = to_bf16_bits(rng.standard_normal((n, HK, D)).astype(np.float32))
        v = to_bf16_bits(rng.standard_normal((n, HK, D)).astype(np.float32))
        dev_o.write(so, k, v)
        pa.pa_reshape_and_cache(to_device_values(k, "bf16", DEV), to_device_values(v, "bf16", DEV), kc, vc,
                                torch.from_numpy(slots).to(DEV))

    for s, n in enumerate([37, 300, 16, 129, 450, 5]):
        add(s, n)
    o.fork(1, 100)
    c.fork(1, 100)  # seq 1's blocks are shared: swapping it out copies them, the fork keeps its own
    for s in (1, 3, 4):
        pairs = c.swap_out(s)
        assert [tuple(p) for p in pairs.tolist()] == o.swap_out(s)
        pa.pa_swap_blocks(kc, vc, kh, vh, torch.from_numpy(pairs).to(DEV))
        dev_o.copy_blocks_to(host_o, [tuple(p) for p in pairs.tolist()])
    for s, n in zip(range(6, 10), [200, 333, 64, 90]):  # reuse and overwrite the freed device blocks
        add(s, n)
    for s in (4, 1):
        pairs = c.swap_in(s)
        assert [tuple(p) for p in pairs.tolist()] == o.swap_in(s)
        pa.pa_swap_blocks(kh, vh, kc, vc, torch.from_numpy(pairs).to(DEV))
        host_o.copy_blocks_to(dev_o, [tuple(p) for p in pairs.tolist()])
    torch.cuda.synchronize()
    check_status_clean()
    o.check_invariants()

    live = [s for s in (0, 1, 2, 4, 5, 6, 7, 8, 9, 100)]
    max_nb = max(c.length(s) for s in live) // BS + 1
    tables, lens = c.block_tables(live, max_nb)
    assert np.array_equal(tables, block_table_array(o, live, max_nb))
    # cache bytes of every block a live sequence reads
    khr, vhr = to_host_raw(kc, "bf16"), to_host_raw(vc, "bf16")
    for b in set(int(x) for x in tables.reshape(-1) if x >= 0):
        wr = dev_o.written(b)
        assert np.array_equal(khr[b][:, wr], dev_o.k_page(b)[:, wr]) and np.array_equal(vhr[b][:, wr],
                                                                                        dev_o.v_page(b)[:, wr])
    q = to_bf16_bits(rng.standard_normal((len(live), H, D)).astype(np.float32))
    out = torch.empty(len(live), H, D, dtype=torch.bfloat16, device=DEV)
    ws = torch.zeros(pa.pa_decode_workspace_bytes(len(live), H, HK, D, max_nb, 0), dtype=torch.uint8, device=DEV)
    pa.pa_decode(out, to_device_values(q, "bf16", DEV), kc, vc, torch.from_numpy(tables).to(DEV),
                 torch.from_numpy(lens).to(DEV), 1 / math.sqrt(D), HK, workspace=ws)
    check_status_clean()
    ref = paged_decode(q, dev_o, tables, lens, 1 / math.sqrt(D))
    assert float(np.max(np.abs(widen(to_host_raw(out, "bf16"), "bf16") - ref))) <= 1e-2


def test_swap_refuses_pageable_host_memory():
    kc = torch.empty(4, HK, BS, D, dtype=torch.bfloat16, device=DEV)
    pageable = torch.empty(4, HK, BS, D, dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device=DEV)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_swap_blocks(kc, kc, pageable, pageable, pairs)
    assert e.value.status == 1
    check_status_clean()
