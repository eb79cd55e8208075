"""pa_decode_no_alloc — paged decode for callers that cannot hand the library
device scratch (a host framework that owns every device allocation and gives
plugins no scratch buffer, or a serving loop that must not call cudaMalloc
because it can synchronise the device).  Its split scratch is a fixed array
inside the library.

Both entry points run the same kernels with the same launch plan; only the
address of the split scratch differs.  So the no-scratch output must equal
pa_decode's bit for bit, on two calls in a row (the array keeps the previous
call's contents, which must not leak into the next result), and both must
match the fp64 oracle within the bf16 bar (max-abs 1e-2).

This file is named to be collected last, and needs nothing from the other
test files, so it passes alone in a fresh process as well as after them.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from oracle.attention import paged_decode, widen
from oracle.cache import PagedKVCache

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 1e-2


def _bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _paged_batch(seed, ctxs, H, Hkv, D=128):
    """A bf16 paged batch on the device (written through pa_reshape_and_cache)
    and the oracle's copy of the same cache."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    nbs = [-(-c // 16) for c in ctxs]
    NB = sum(nbs) + 5
    max_nb = max(nbs) + 2
    perm = torch.randperm(NB, generator=g)
    tables = torch.full((len(ctxs), max_nb), -1, dtype=torch.int32)
    slots, off = [], 0
    for i, (c, n) in enumerate(zip(ctxs, nbs)):
        tables[i, :n] = perm[off:off + n].to(torch.int32)
        off += n
        slots += [int(tables[i, t // 16]) * 16 + t % 16 for t in range(c)]
    T = len(slots)
    kc = torch.zeros(NB, Hkv, 16, D, dtype=torch.bfloat16, device=DEV)
    vc = torch.zeros_like(kc)
    key = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    value = torch.randn(T, Hkv, D, generator=g).to(torch.bfloat16)
    pa.pa_reshape_and_cache(key.to(DEV), value.to(DEV), kc, vc, torch.tensor(slots, dtype=torch.int64, device=DEV))
    q = torch.randn(len(ctxs), H, D, generator=g).to(torch.bfloat16)
    oracle_cache = PagedKVCache(NB, Hkv, D, 16, "bf16")
    oracle_cache.write(slots, _bits(key), _bits(value))
    host = {"q": _bits(q), "cache": oracle_cache, "tables": tables.numpy(), "ctxs": list(ctxs)}
    return q.to(DEV), kc, vc, tables.to(DEV), torch.tensor(ctxs, dtype=torch.int32, device=DEV), host


@pytest.mark.parametrize("partition_tokens", [0, 512, -1])
def test_no_alloc_matches_workspace_decode_twice(partition_tokens):
    q, kc, vc, bt, cl, host = _paged_batch(7, [1, 17, 300, 2048, 913, 64, 5000, 33], 32, 8)
    scale = 1.0 / math.sqrt(128)
    B, H, D = q.shape
    n = pa.pa_decode_workspace_bytes(B, H, 8, D, bt.shape[1], partition_tokens)
    ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=DEV) if n else None
    ref = torch.empty_like(q)
    pa.pa_decode(ref, q, kc, vc, bt, cl, scale, 8, workspace=ws, partition_tokens=partition_tokens)
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        pa.pa_decode_no_alloc(out, q, kc, vc, bt, cl, scale, 8, partition_tokens=partition_tokens)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(out), _bits(ref)), call
    exact = paged_decode(host["q"], host["cache"], host["tables"], host["ctxs"], scale)
    err = float(np.max(np.abs(widen(_bits(out), "bf16") - exact)))
    assert err <= TOL_BF16, err
    st, bits = pa.pa_get_device_status()
    assert st == 0 and bits == 0


def test_no_alloc_after_a_different_shape():
    """A smaller call after a larger one: leftovers of the first must not
    reach the second."""
    scale = 1.0 / math.sqrt(128)
    for seed, ctxs in ((11, [4000, 3000, 2000, 100]), (12, [50, 700])):
        q, kc, vc, bt, cl, _ = _paged_batch(seed, ctxs, 16, 4)
        B, H, D = q.shape
        n = pa.pa_decode_workspace_bytes(B, H, 4, D, bt.shape[1], 0)
        ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
        ref = torch.empty_like(q)
        pa.pa_decode(ref, q, kc, vc, bt, cl, scale, 4, workspace=ws)
        out = torch.empty_like(q)
        pa.pa_decode_no_alloc(out, q, kc, vc, bt, cl, scale, 4)
        torch.cuda.synchronize()
        assert np.array_equal(_bits(out), _bits(ref))


def test_no_alloc_rejects_split_beyond_its_buffer():
    """16-token partitions of 64 x 32 heads x 512 blocks need ~0.5 GB of
    partials: refused before any launch."""
    B, H, Hkv, D, max_nb = 64, 32, 8, 128, 512
    assert pa.pa_decode_workspace_bytes(B, H, Hkv, D, max_nb, 16) > pa.NO_ALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, D, dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros(4, Hkv, 16, D, dtype=torch.bfloat16, device=DEV)
    bt = torch.zeros(B, max_nb, dtype=torch.int32, device=DEV)
    cl = torch.ones(B, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    with pytest.raises(pa.PagedAttentionError) as e:
        pa.pa_decode_no_alloc(out, q, kc, kc, bt, cl, 0.1, Hkv, partition_tokens=16)
    assert e.value.status == 7
