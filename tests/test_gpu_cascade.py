"""GPU parity of the shared-prefix decode (pa_decode_cascade) against the
fp64 oracle.

Batches of prompts forked into samples (forks of forks too) are built
through the library's allocator, copy-on-write copies and cache writes; the
groups come from the allocator (pa_alloc_prefix_groups).  The output must
match the plain definition of attention (oracle.attention.paged_decode)
within 1e-2 (bf16) / 1e-5 (fp32) in both split modes.  Malformed groups
(not tiling the batch, too many members, more shared blocks than a member
holds) must be reported in the status word and still give the right
output, because the kernels then decode those sequences in full.
"""

import math

import numpy as np
import pytest
import torch

import paged_kv_cache_351_b200 as pa
from gpu_harness import TOL, to_device_values, to_host_raw
from oracle.attention import paged_decode, widen
from oracle.cache import PagedKVCache

pytestmark = pytest.mark.gpu
DEV = "cuda"
BS = 16
TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def _store(x, dtype):
    from workloads import to_bf16_bits

    x = np.asarray(x, np.float32)
    return x if dtype == "f32" else to_bf16_bits(x)


class Forest:
    """Prompts forked into samples on the device and in the oracle."""

    def __init__(self, seed, n_prompts, samples, H, Hkv, D, dtype, max_len=700, max_app=40, forks_of_forks=False,
                 exact_prompts=False, empty_seqs=0):
        rng = np.random.default_rng(seed)
        self.H, self.Hkv, self.D, self.dtype = H, Hkv, D, dtype
        lens = rng.integers(1, max_len, size=n_prompts)
        if exact_prompts:
            lens = (lens // BS + 1) * BS
        nb = int(sum(-(-int(l) // BS) for l in lens) * (samples + 1) + (max_app // BS + 2) * n_prompts * samples + 64)
        self.nb = nb
        order = rng.permutation(nb).astype(np.int32)
        self.alloc = pa.Allocator(nb, BS, order)
        self.cache = PagedKVCache(nb, Hkv, D, BS, dtype)
        tdt = TORCH_DT[dtype]
        self.kc = torch.full((nb, Hkv, BS, D), float("nan"), dtype=tdt, device=DEV)
        self.vc = torch.full((nb, Hkv, BS, D), float("nan"), dtype=tdt, device=DEV)

        def append(seq, n):
            slots, cow = self.alloc.append(seq, n)
            if cow:
                self.cache.copy_blocks(cow)
                pa.pa_copy_blocks(self.kc, self.vc, torch.tensor(cow, dtype=torch.int64, device=DEV))
            if n:
                k = _store(rng.standard_normal((n, Hkv, D)), dtype)
                v = _store(rng.standard_normal((n, Hkv, D)), dtype)
                self.cache.write(slots, k, v)
                pa.pa_reshape_and_cache(to_device_values(k, dtype, DEV), to_device_values(v, dtype, DEV), self.kc,
                                        self.vc, torch.from_numpy(slots).to(DEV))

        self.batch, sid = [], 0
        for p in range(n_prompts):
            root = sid
            sid += 1
            self.alloc.add(root)
            append(root, int(lens[p]))
            members = [root]
            for _ in range(samples - 1):
                parent = members[int(rng.integers(0, len(members)))] if forks_of_forks else root
                self.alloc.fork(parent, sid)
                members.append(sid)
                sid += 1
                if forks_of_forks:
                    append(sid - 1, int(rng.integers(0, max_app)))
            for k, m in enumerate(members):
                # with exact_prompts the prompt's own sequence appends nothing
                append(m, 0 if (exact_prompts and k == 0) else int(rng.integers(1, max_app)))
            self.batch += members
        for _ in range(empty_seqs):
            self.alloc.add(sid)
            self.batch.insert(int(rng.integers(0, len(self.batch) + 1)), sid)
            sid += 1
        self.max_nb = max(self.alloc.length(s) for s in self.batch) // BS + 2
        tables, lens_ = self.alloc.block_tables(self.batch, self.max_nb)
        self.tables, self.lens = tables, lens_
        self.bt = torch.from_numpy(tables).to(DEV)
        self.cl = torch.from_numpy(lens_).to(DEV)
        self.q = _store(rng.standard_normal((len(self.batch), H, D)), dtype)
        self.qd = to_device_values(self.q, dtype, DEV)
        self.scale = 1.0 / math.sqrt(D)

    def groups(self, max_group_size):
        gs, gb = self.alloc.prefix_groups(self.batch, max_group_size)
        return torch.from_numpy(np.ascontiguousarray(gs)).to(DEV), torch.from_numpy(np.ascontiguousarray(gb)).to(DEV)

    def run(self, gs, gb, max_group_size, mode=0):
        out = torch.empty_like(self.qd)
        n = pa.pa_decode_cascade_workspace_bytes(len(self.batch), self.H, self.Hkv, self.D, max_group_size, mode)
        ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
        pa.pa_decode_cascade(out, self.qd, self.kc, self.vc, self.bt, self.cl, gs, gb, max_group_size, self.scale,
                             self.Hkv, ws, partition_tokens=mode)
        torch.cuda.synchronize()
        assert int(ws[:pa.PA_DECODE_WS_HEADER_BYTES].count_nonzero()) == 0
        return out

    def err(self, out):
        ref = paged_decode(self.q, self.cache, self.tables, self.lens, self.scale)
        got = widen(to_host_raw(out, self.dtype), self.dtype)
        return float(np.max(np.abs(got - ref)))


def _status():
    return pa.pa_get_device_status()


@pytest.mark.parametrize("H,Hkv,M", [(8, 8, 4), (8, 8, 8), (16, 8, 4), (32, 8, 2), (8, 8, 1)])
@pytest.mark.parametrize("mode", [0, -1])
def test_cascade_parity_bf16(H, Hkv, M, mode):
    f = Forest(10 + H + M, 12, M, H, Hkv, 128, "bf16")
    gs, gb = f.groups(M)
    if M > 1:
        assert int(gb.sum()) > 0
    out = f.run(gs, gb, M, mode)
    assert _status() == (0, 0)
    assert not torch.isnan(out.float()).any()
    assert f.err(out) <= TOL["bf16"]


def test_cascade_parity_fp32():
    f = Forest(3, 10, 4, 8, 8, 64, "f32")
    gs, gb = f.groups(4)
    for mode in (0, -1):
        out = f.run(gs, gb, 4, mode)
        assert _status() == (0, 0)
        assert f.err(out) <= TOL["f32"]


def test_cascade_forks_of_forks_and_empty_sequences():
    f = Forest(4, 10, 4, 16, 8, 128, "bf16", forks_of_forks=True, empty_seqs=3)
    gs, gb = f.groups(4)
    out = f.run(gs, gb, 4)
    assert _status() == (0, 0)
    assert f.err(out) <= TOL["bf16"]
    assert torch.all(out[[f.batch.index(s) for s in f.batch if f.alloc.length(s) == 0]] == 0)


def test_cascade_members_with_nothing_past_the_prefix():
    """Prompts of whole blocks, samples that append nothing: their output is
    the shared prefix's result alone."""
    f = Forest(5, 8, 4, 8, 8, 128, "bf16", exact_prompts=True)
    gs, gb = f.groups(4)
    assert any(f.alloc.length(s) == int(gb[v]) * BS for v in range(len(gb))
               for s in f.batch[int(gs[v]):int(gs[v + 1])])
    for mode in (0, -1):
        out = f.run(gs, gb, 4, mode)
        assert _status() == (0, 0)
        assert f.err(out) <= TOL["bf16"]


def test_cascade_matches_decode_on_a_single_group_batch():
    """One group: every sequence a sample of the same prompt."""
    f = Forest(6, 1, 8, 8, 8, 128, "bf16", max_len=3000)
    gs, gb = f.groups(8)
    assert len(gb) == 1 and int(gb[0]) > 0
    out = f.run(gs, gb, 8)
    assert _status() == (0, 0)
    assert f.err(out) <= TOL["bf16"]


def test_cascade_malformed_groups_fall_back_to_full_decode():
    f = Forest(7, 6, 4, 8, 8, 128, "bf16")
    gs, gb = f.groups(4)
    B = len(f.batch)
    # groups that do not tile the batch: reported, every sequence decoded in full
    bad = gs.clone()
    bad[-1] = B - 1
    out = f.run(bad, gb, 4)
    st, bits = _status()
    assert bits & pa.PA_DEV_BAD_CONTEXT
    assert f.err(out) <= TOL["bf16"]
    # more shared blocks than the members hold: capped and reported
    big = gb.clone()
    big[0] += 1000
    out = f.run(gs, big, 4)
    st, bits = _status()
    assert bits & pa.PA_DEV_BAD_CONTEXT
    assert f.err(out) <= TOL["bf16"]
    # a group larger than max_group_size: decoded in full and reported
    gs2, gb2 = f.groups(8)
    if int((gs2[1:] - gs2[:-1]).max()) > 2:
        out = f.run(gs2, gb2, 2)
        st, bits = _status()
        assert bits & pa.PA_DEV_BAD_CONTEXT
        assert f.err(out) <= TOL["bf16"]


def test_cascade_rejects_bad_arguments():
    f = Forest(8, 2, 2, 8, 8, 128, "bf16")
    gs, gb = f.groups(2)
    out = torch.empty_like(f.qd)
    n = pa.pa_decode_cascade_workspace_bytes(len(f.batch), 8, 8, 128, 2, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    with pytest.raises(pa.PagedAttentionError) as e:  # G * max_group_size = 3
        pa.pa_decode_cascade(out, f.qd, f.kc, f.vc, f.bt, f.cl, gs, gb, 3, f.scale, 8, ws)
    assert e.value.status == 2
    with pytest.raises(pa.PagedAttentionError) as e:  # workspace too small
        pa.pa_decode_cascade(out, f.qd, f.kc, f.vc, f.bt, f.cl, gs, gb, 2, f.scale, 8, ws[: n // 2])
    assert e.value.status == 1
    with pytest.raises(pa.PagedAttentionError) as e:  # fixed partitions
        pa.pa_decode_cascade(out, f.qd, f.kc, f.vc, f.bt, f.cl, gs, gb, 2, f.scale, 8, ws, partition_tokens=512)
    assert e.value.status == 2
    with pytest.raises(pa.PagedAttentionError) as e:  # group_start of the wrong length
        pa.pa_decode_cascade(out, f.qd, f.kc, f.vc, f.bt, f.cl, gs[:-1], gb, 2, f.scale, 8, ws)
    assert e.value.status == 1
