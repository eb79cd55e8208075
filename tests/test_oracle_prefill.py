"""Pins of the multi-token (chunked-prefill) attention oracle.

Each pin checks the oracle against something other than itself:
* every row equals the decode oracle (pinned on its own against torch SDPA
  and closed forms) run over the context truncated at that row's position;
* a batch of single-token requests equals the decode oracle;
* a whole prompt (no prior context) equals torch's fp64 SDPA with
  ``is_causal=True`` (torch builds the causal mask itself);
* a chunk over a prior context equals torch's fp64 SDPA with a mask built
  by ``tril`` with the prior length as diagonal offset;
* scalar ``math`` brute force on tiny sizes;
* bitwise invariance under a permutation of the physical blocks;
* planted mistakes (causal offset without the prior context, strict mask,
  wrong head map, missing scale) each fail at least one pin.
"""

import math

import numpy as np
import pytest
import torch

import oracle.prefill as prefill
from oracle.attention import paged_decode
from oracle.cache import PagedKVCache
from workloads import to_bf16_bits

BS = 16


class Case:
    """Random paged state: sequences (prior, n) with their K/V in permuted
    blocks of an oracle cache, and n query rows each."""

    def __init__(self, seed, pairs, H, hk, D, dtype="f32", perm=None):
        rng = np.random.default_rng(seed)
        self.pairs = list(pairs)
        self.H, self.hk, self.D, self.dtype = H, hk, D, dtype
        self.ctx = np.array([a + b for a, b in pairs], np.int64)
        self.qlen = np.array([b for _, b in pairs], np.int64)
        self.qs = np.concatenate([[0], np.cumsum(self.qlen)]).astype(np.int64)
        nbs = [-(-int(c) // BS) for c in self.ctx]
        self.NB = sum(nbs) + 3
        order = rng.permutation(self.NB)  # drawn either way, so the values below do not depend on perm
        if perm is not None:
            order = perm
        self.order = order
        self.max_nb = max(1, max(nbs))
        self.tables = np.full((len(pairs), self.max_nb), -1, np.int64)
        off = 0
        for i, n in enumerate(nbs):
            self.tables[i, :n] = order[off:off + n]
            off += n
        self.cache = PagedKVCache(self.NB, hk, D, BS, dtype)
        self.kv = []
        for i, c in enumerate(self.ctx.tolist()):
            k = rng.standard_normal((c, hk, D)).astype(np.float32)
            v = rng.standard_normal((c, hk, D)).astype(np.float32)
            if dtype == "bf16":
                k, v = to_bf16_bits(k), to_bf16_bits(v)
            slots = [int(self.tables[i, t // BS]) * BS + t % BS for t in range(c)]
            self.cache.write(slots, k, v)
            self.kv.append((k, v))
        q = rng.standard_normal((int(self.qs[-1]), H, D)).astype(np.float32)
        self.q = to_bf16_bits(q) if dtype == "bf16" else q
        self.scale = 1.0 / math.sqrt(D)

    def widen(self, x):
        from oracle.attention import widen

        return widen(x, self.dtype)

    def run(self):
        return prefill.paged_prefill(self.q, self.cache, self.tables, self.ctx, self.qs, self.scale)


PAIRS = [(0, 1), (0, 17), (23, 7), (0, 40), (16, 16), (33, 20), (5, 0), (0, 0), (47, 1)]


def _pin_rows_are_truncated_decodes(case):
    out = case.run()
    for i, (prior, n) in enumerate(case.pairs):
        for j in range(n):
            r = int(case.qs[i]) + j
            ref = paged_decode(case.q[r:r + 1], case.cache, case.tables[i:i + 1], [prior + j + 1], case.scale)
            assert np.max(np.abs(out[r] - ref[0])) <= 1e-12, (i, j)


def _pin_torch_sdpa(case):
    out = case.run()
    G = case.H // case.hk
    for i, (prior, n) in enumerate(case.pairs):
        if n == 0:
            continue
        k, v = case.kv[i]
        kt = torch.from_numpy(case.widen(k)).permute(1, 0, 2)[None]  # [1, hk, ctx, D]
        vt = torch.from_numpy(case.widen(v)).permute(1, 0, 2)[None]
        a = int(case.qs[i])
        qt = torch.from_numpy(case.widen(case.q[a:a + n])).permute(1, 0, 2)[None]  # [1, H, n, D]
        if prior == 0:
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=case.scale,
                                                                   enable_gqa=G > 1)
        else:
            mask = torch.ones(n, prior + n, dtype=torch.bool).tril(diagonal=prior)
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=case.scale,
                                                                   enable_gqa=G > 1)
        ref = ref[0].permute(1, 0, 2).numpy()
        assert np.max(np.abs(out[a:a + n] - ref)) <= 1e-12, i


def _pin_brute_force():
    case = Case(3, [(0, 3), (2, 3), (4, 1)], H=2, hk=1, D=3)
    out = case.run()
    for i, (prior, n) in enumerate(case.pairs):
        k, v = case.kv[i]
        for j in range(n):
            r = int(case.qs[i]) + j
            for h in range(2):
                s = [case.scale * sum(float(case.q[r, h, d]) * float(k[t, 0, d]) for d in range(3))
                     for t in range(prior + j + 1)]
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                z = sum(w)
                for d in range(3):
                    ref = sum(w[t] * float(v[t, 0, d]) for t in range(len(s))) / z
                    assert abs(out[r, h, d] - ref) <= 1e-12


def test_rows_are_truncated_decodes():
    _pin_rows_are_truncated_decodes(Case(1, PAIRS, H=4, hk=2, D=8))


def test_single_token_requests_equal_decode():
    pairs = [(c - 1, 1) for c in (1, 2, 16, 17, 40, 100)]
    case = Case(2, pairs, H=6, hk=3, D=16, dtype="bf16")
    ref = paged_decode(case.q, case.cache, case.tables, case.ctx, case.scale)
    assert np.max(np.abs(case.run() - ref)) <= 1e-12


def test_matches_torch_sdpa():
    _pin_torch_sdpa(Case(4, PAIRS, H=8, hk=2, D=32))
    _pin_torch_sdpa(Case(5, [(0, 50), (70, 33)], H=4, hk=4, D=16, dtype="bf16"))


def test_brute_force_tiny():
    _pin_brute_force()


def test_block_permutation_invariance():
    a = Case(6, PAIRS, H=4, hk=2, D=8)
    b = Case(6, PAIRS, H=4, hk=2, D=8, perm=np.random.default_rng(9).permutation(a.NB))
    assert not np.array_equal(a.tables, b.tables)
    assert np.array_equal(a.run(), b.run())


def test_rejects_more_new_tokens_than_context():
    case = Case(7, [(0, 4)], H=2, hk=1, D=4)
    with pytest.raises(ValueError):
        prefill.paged_prefill(case.q, case.cache, case.tables, [3], case.qs, case.scale)


# -- planted mistakes ----------------------------------------------------------

def _mutant_no_prior(q, k, v, prior, scale):
    return _ORIG(q, k, v, 0, scale)  # row j sees keys 0 .. j, ignoring the prior context


def _mutant_strict(q, k, v, prior, scale):
    n, h_q, d = q.shape
    out = np.zeros((n, h_q, d))
    for j in range(n):
        pos = prior + j
        if pos == 0:
            continue
        out[j:j + 1] = _ORIG(q[j:j + 1], k[:pos], v[:pos], pos - 1, scale)
    return out


def _mutant_head_map(q, k, v, prior, scale):
    n, h_q, d = q.shape
    hk = k.shape[1]
    kk = np.stack([k[:, h % hk] for h in range(h_q)], axis=1)
    vv = np.stack([v[:, h % hk] for h in range(h_q)], axis=1)
    return _ORIG(q, kk, vv, prior, scale)


def _mutant_no_scale(q, k, v, prior, scale):
    return _ORIG(q, k, v, prior, 1.0)


_ORIG = prefill._rows_of_sequence


@pytest.mark.parametrize("mutant", [_mutant_no_prior, _mutant_strict, _mutant_head_map, _mutant_no_scale])
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    monkeypatch.setattr(prefill, "_rows_of_sequence", mutant)
    caught = 0
    for pin in (lambda: _pin_rows_are_truncated_decodes(Case(1, PAIRS, H=4, hk=2, D=8)),
                lambda: _pin_torch_sdpa(Case(4, PAIRS, H=8, hk=2, D=32)),
                _pin_brute_force):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1
