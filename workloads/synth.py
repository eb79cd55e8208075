"""Seeded synthetic workloads shaped like the LLaMA-7B/13B serving batches that
the PagedAttention pages measure on (vLLM launch blog, "performance" section:
LLaMA-7B on A10G, LLaMA-13B on A100-40GB, lengths sampled from ShareGPT).

No dataset is used: lognormal and uniform length draws stand in for the
ShareGPT length mix.  Every value is drawn from ``numpy.random.default_rng``
seeded by ``SeedSequence([351 + index, tag, ...])`` so that any chunk of any
token stream can be regenerated on its own (the oracle recomputes sampled
rows of the full-size workloads without materialising the whole batch).

Nothing here implements the method: the allocator operations are *requests*
(add a sequence, append n tokens, fork), not their effect on block tables.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Tuple, Union

import numpy as np

BLOCK_SIZE = 16
_BASE_SEED = 351

# Tags that separate the independent random streams of one workload.
_TAG_CTX = 1
_TAG_PERM = 2
_TAG_K = 3
_TAG_V = 4
_TAG_Q = 5
_TAG_OUTLIER = 6
_TAG_PROMPT = 7
_TAG_APPEND = 8

# Token values are generated in chunks of this many positions, each chunk from
# its own seed, so that a slice of a long stream costs only its own chunks.
_CHUNK = 1024


@dataclass(frozen=True)
class Workload:
    """Shape of one paged-decode workload (one attention layer)."""

    name: str
    index: int  # position in the config list; seed = 351 + index
    dtype: str  # "f32" or "bf16": the KV / query / output storage type
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int = BLOCK_SIZE
    description: str = ""
    kv_dtype: str = ""  # cache storage type when it differs from dtype ("fp8": e4m3 codes + per-head scales)

    @property
    def seed(self) -> int:
        return _BASE_SEED + self.index

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def cache_dtype(self) -> str:
        return self.kv_dtype or self.dtype

    @property
    def cache_elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2, "fp8": 1}[self.cache_dtype]


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny_fp32", 0, "f32", 8, 8, 64,
                 description="4 seqs ctx {1,17,33,100}, H=H_kv=8, D=64, fp32, 64 permuted blocks"),
        Workload("llama7b_bs64", 1, "bf16", 32, 32, 128,
                 description="B=64, H=H_kv=32, D=128, bf16, ctx lognormal(median 512, sigma 0.75) "
                             "clipped [16,2048], 40 GB pool (152,587 blocks)"),
        Workload("gqa_bs256", 2, "bf16", 32, 8, 128,
                 description="B=256, H=32 on H_kv=8, D=128, bf16, ctx lognormal(median 1024, sigma 0.75) "
                             "clipped [32,8192], 10 K outlier channels x8"),
        Workload("parallel_sampling_13b", 3, "bf16", 40, 40, 128,
                 description="64 prompts U{256..1024} x 4 forked samples, each +U{1..64} tokens, "
                             "H=H_kv=40, D=128, bf16"),
        Workload("long_ctx_splitk", 4, "bf16", 32, 8, 128,
                 description="B=8, ctx {32,48,64,80,96,112,128,128}k, H=32 on H_kv=8, D=128, bf16, "
                             "512-token partitions + LSE reduce"),
        # FP8 KV-cache variants: same seeds, lengths and bf16 token values; the
        # cache stores e4m3 codes with per-kv-head scales (kv_scales).
        Workload("llama7b_bs64_fp8", 1, "bf16", 32, 32, 128, kv_dtype="fp8",
                 description="llama7b_bs64 with an e4m3 KV cache (per-head scales), bf16 query/output"),
        Workload("gqa_bs256_fp8", 2, "bf16", 32, 8, 128, kv_dtype="fp8",
                 description="gqa_bs256 with an e4m3 KV cache (per-head scales), bf16 query/output"),
        # Multi-token (chunked-prefill) steps: each sequence appends q_len
        # tokens at once and every new token is a query row (causal).
        Workload("prefill_tiny", 7, "bf16", 4, 2, 128,
                 description="11 seqs of (prior context, new tokens) edge cases incl. empty and decode rows, "
                             "H=4 on H_kv=2, D=128, bf16"),
        Workload("prefill_chunks_llama7b", 8, "bf16", 32, 32, 128,
                 description="16 prefill chunks of 512 tokens over prior contexts U{0..3584}, H=H_kv=32, "
                             "D=128, bf16"),
        Workload("prefill_mixed_gqa", 9, "bf16", 32, 8, 128,
                 description="4 prefill chunks of 512 tokens (prior U{0..7680}) mixed with 60 decode rows "
                             "(ctx lognormal median 1024), H=32 on H_kv=8, D=128, bf16"),
    )
}


def workload_by_name(name: str) -> Workload:
    return WORKLOADS[name]


def _rng(w: Workload, *tags: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, *[int(t) for t in tags]]))


# --------------------------------------------------------------------------
# bf16 storage helpers (input preparation only)
# --------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to bfloat16, nearest-even; return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(w: Workload, x: np.ndarray) -> np.ndarray:
    """float32 draws -> the workload's storage form (float32, or bf16 bits)."""
    if w.dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    return to_bf16_bits(x)


# --------------------------------------------------------------------------
# allocator requests
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class AddOp:
    seq: int


@dataclass(frozen=True)
class ForkOp:
    parent: int
    child: int


@dataclass(frozen=True)
class AppendOp:
    """Append ``n`` tokens to ``seq``; their K/V are positions
    ``[start, start+n)`` of token stream ``stream``."""

    seq: int
    n: int
    stream: int
    start: int


Op = Union[AddOp, ForkOp, AppendOp]


@dataclass
class Plan:
    """Everything that defines one workload instance."""

    workload: Workload
    num_blocks: int
    free_order: np.ndarray  # int32 permutation: blocks in the order they are handed out
    setup_ops: List[Op]  # requests before the decode step (prefill, forks, earlier appends)
    step_ops: List[Op]  # requests of the decode step itself (one new token per sequence)
    batch: np.ndarray  # int64 sequence ids in batch order
    context_lens: np.ndarray  # int32 context length of each batch sequence after the step
    outlier_channels: np.ndarray = field(default_factory=lambda: np.zeros((0, 2), np.int64))
    # parallel sampling only: ops after the first append round (for a mid-replay check)
    first_round_end: int = -1
    # new tokens of each batch sequence in the step (1 for a decode step); the
    # step's query rows are these tokens, sequence by sequence
    query_lens: np.ndarray = None

    def __post_init__(self):
        if self.query_lens is None:
            self.query_lens = np.ones(len(self.context_lens), np.int32)

    @property
    def num_query_rows(self) -> int:
        return int(np.sum(self.query_lens))

    @property
    def query_start(self) -> np.ndarray:
        """int32 [B + 1]: row offset of each sequence's queries."""
        return np.concatenate([[0], np.cumsum(self.query_lens)]).astype(np.int32)

    @property
    def B(self) -> int:
        return int(self.batch.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        bs = self.workload.block_size
        return int(max(1, max((int(c) + bs - 1) // bs for c in self.context_lens)))


def _lognormal_lengths(w: Workload, n: int, median: float, sigma: float, lo: int, hi: int) -> np.ndarray:
    r = _rng(w, _TAG_CTX)
    x = np.exp(r.normal(math.log(median), sigma, size=n))
    return np.clip(np.rint(x), lo, hi).astype(np.int32)


def _single_plan(w: Workload, ctx: np.ndarray, num_blocks: int) -> Plan:
    """Independent sequences: prefill ctx-1 tokens, then the step appends one."""
    setup: List[Op] = []
    step: List[Op] = []
    for i, c in enumerate(ctx.tolist()):
        setup.append(AddOp(i))
        if c > 1:
            setup.append(AppendOp(i, c - 1, i, 0))
    for i, c in enumerate(ctx.tolist()):
        if c > 0:
            step.append(AppendOp(i, 1, i, c - 1))
    order = _rng(w, _TAG_PERM).permutation(num_blocks).astype(np.int32)
    return Plan(w, num_blocks, order, setup, step, np.arange(len(ctx), dtype=np.int64), ctx.astype(np.int32))


def _prefill_plan(w: Workload, prior: np.ndarray, qlen: np.ndarray, spare: float = 1.25) -> Plan:
    """Sequence i holds prior[i] tokens before the step (stream i, positions
    [0, prior)) and appends qlen[i] tokens in it (positions [prior, prior+qlen))."""
    setup: List[Op] = []
    step: List[Op] = []
    for i, (c, q) in enumerate(zip(prior.tolist(), qlen.tolist())):
        setup.append(AddOp(i))
        if c > 0:
            setup.append(AppendOp(i, c, i, 0))
    for i, (c, q) in enumerate(zip(prior.tolist(), qlen.tolist())):
        if q > 0:
            step.append(AppendOp(i, q, i, c))
    ctx = (prior + qlen).astype(np.int32)
    nb = max(1, int(math.ceil(spare * _blocks_needed(ctx, w.block_size))))
    order = _rng(w, _TAG_PERM).permutation(nb).astype(np.int32)
    return Plan(w, nb, order, setup, step, np.arange(len(ctx), dtype=np.int64), ctx,
                query_lens=qlen.astype(np.int32))


def _blocks_needed(ctx: np.ndarray, bs: int) -> int:
    return int(sum((int(c) + bs - 1) // bs for c in ctx))


def make_plan(w: Union[Workload, str]) -> Plan:
    """Build the seeded instance of a named workload."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    if w.kv_dtype == "fp8":
        base = make_plan(w.name[: -len("_fp8")])
        base.workload = w
        if w.name.startswith("llama7b"):
            # the same 40 GB of pool, now of 1-byte elements
            base.num_blocks = int(40_000_000_000 // (2 * w.num_kv_heads * w.block_size * w.head_size))
            base.free_order = _rng(w, _TAG_PERM).permutation(base.num_blocks).astype(np.int32)
        return base
    bs = w.block_size
    if w.name == "tiny_fp32":
        ctx = np.array([1, 17, 33, 100], np.int32)
        return _single_plan(w, ctx, 64)
    if w.name == "llama7b_bs64":
        ctx = _lognormal_lengths(w, 64, 512.0, 0.75, 16, 2048)
        # a 40 GB pool for K+V: 40e9 // (2 * H_kv * bs * D * 2 bytes)
        nb = 40_000_000_000 // (2 * w.num_kv_heads * bs * w.head_size * w.elem_bytes)
        return _single_plan(w, ctx, int(nb))
    if w.name == "gqa_bs256":
        ctx = _lognormal_lengths(w, 256, 1024.0, 0.75, 32, 8192)
        plan = _single_plan(w, ctx, int(math.ceil(1.25 * _blocks_needed(ctx, bs))))
        r = _rng(w, _TAG_OUTLIER)
        n_ch = w.num_kv_heads * w.head_size
        n_out = int(round(0.01 * n_ch))
        flat = np.sort(r.choice(n_ch, size=n_out, replace=False))
        plan.outlier_channels = np.stack([flat // w.head_size, flat % w.head_size], axis=1).astype(np.int64)
        return plan
    if w.name == "long_ctx_splitk":
        ctx = (np.array([32, 48, 64, 80, 96, 112, 128, 128], np.int32) * 1024).astype(np.int32)
        return _single_plan(w, ctx, int(math.ceil(1.25 * _blocks_needed(ctx, bs))))
    if w.name == "parallel_sampling_13b":
        return _parallel_sampling_plan(w)
    if w.name == "prefill_tiny":
        pairs = [(0, 1), (0, 17), (23, 7), (0, 300), (16, 16), (100, 129), (511, 1), (257, 256), (40, 0), (0, 0),
                 (5, 33)]
        prior = np.array([a for a, _ in pairs], np.int32)
        qlen = np.array([b for _, b in pairs], np.int32)
        return _prefill_plan(w, prior, qlen, spare=1.5)
    if w.name == "prefill_chunks_llama7b":
        prior = _rng(w, _TAG_CTX).integers(0, 3584, size=16, endpoint=True).astype(np.int32)
        return _prefill_plan(w, prior, np.full(16, 512, np.int32))
    if w.name == "prefill_mixed_gqa":
        r = _rng(w, _TAG_CTX)
        prior_chunks = r.integers(0, 7680, size=4, endpoint=True).astype(np.int32)
        dec = np.clip(np.rint(np.exp(r.normal(math.log(1024.0), 0.75, size=60))), 32, 8192).astype(np.int32)
        prior = np.concatenate([prior_chunks, dec - 1]).astype(np.int32)
        qlen = np.concatenate([np.full(4, 512, np.int32), np.ones(60, np.int32)])
        return _prefill_plan(w, prior, qlen)
    raise KeyError(w.name)


N_PROMPTS = 64
N_SAMPLES = 4


def _parallel_sampling_plan(w: Workload) -> Plan:
    """64 prompts, each prefilled then forked into 4 samples that share the
    prompt blocks; the samples append tokens round-robin (step s, prompt p,
    sample j) until each has its own count.  Sample 0 is the prompt's own
    sequence.  Streams: prompt p -> stream p; sample (p, j) -> 64 + 4p + j."""
    bs = w.block_size
    rp = _rng(w, _TAG_PROMPT)
    plen = rp.integers(256, 1024, size=N_PROMPTS, endpoint=True).astype(np.int64)
    ra = _rng(w, _TAG_APPEND)
    napp = ra.integers(1, 64, size=(N_PROMPTS, N_SAMPLES), endpoint=True).astype(np.int64)

    ops: List[Op] = []
    for p in range(N_PROMPTS):
        sid = N_SAMPLES * p
        ops.append(AddOp(sid))
        ops.append(AppendOp(sid, int(plen[p]), p, 0))
        for j in range(1, N_SAMPLES):
            ops.append(ForkOp(sid, sid + j))
    first_round_end = -1
    for s in range(int(napp.max())):
        for p in range(N_PROMPTS):
            for j in range(N_SAMPLES):
                if napp[p, j] > s:
                    ops.append(AppendOp(N_SAMPLES * p + j, 1, N_PROMPTS + N_SAMPLES * p + j, s))
        if s == 0:
            first_round_end = len(ops)
    # Upper bound on the blocks ever in use: each prompt's blocks plus, per
    # sample, one copied partial block and the blocks its own tokens fill.
    bound = int(sum((int(l) + bs - 1) // bs for l in plen)
                + sum(1 + (int(n) + bs - 1) // bs for n in napp.reshape(-1)))
    nb = int(math.ceil(1.25 * bound))
    order = _rng(w, _TAG_PERM).permutation(nb).astype(np.int32)
    batch = np.arange(N_PROMPTS * N_SAMPLES, dtype=np.int64)
    ctx = (plen[:, None] + napp).reshape(-1).astype(np.int32)
    return Plan(w, nb, order, ops, [], batch, ctx, first_round_end=first_round_end)


def parallel_sampling_lengths(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """(prompt lengths [64], appended counts [64, 4]) of the sampling workload."""
    rp = _rng(w, _TAG_PROMPT)
    plen = rp.integers(256, 1024, size=N_PROMPTS, endpoint=True).astype(np.int64)
    ra = _rng(w, _TAG_APPEND)
    napp = ra.integers(1, 64, size=(N_PROMPTS, N_SAMPLES), endpoint=True).astype(np.int64)
    return plen, napp


# --------------------------------------------------------------------------
# token values
# --------------------------------------------------------------------------

def _chunk_values(w: Workload, tag: int, stream: int, chunk: int, outliers: np.ndarray,
                  rows: int = _CHUNK) -> np.ndarray:
    """The first ``rows`` positions of a chunk.  Draws are sequential, so a
    prefix of a chunk equals the same rows of the whole chunk."""
    r = _rng(w, tag, stream, chunk)
    x = r.standard_normal(size=(rows, w.num_kv_heads, w.head_size), dtype=np.float32)
    if tag == _TAG_K and outliers.shape[0]:
        x[:, outliers[:, 0], outliers[:, 1]] *= np.float32(8.0)
    return x


def stream_kv(plan: Plan, stream: int, start: int, n: int) -> Tuple[np.ndarray, np.ndarray]:
    """K and V of positions ``[start, start+n)`` of a token stream, in storage
    form (float32, or bf16 bits as uint16), each shaped [n, H_kv, D]."""
    w = plan.workload
    out = []
    for tag in (_TAG_K, _TAG_V):
        if n <= 0:
            shape = (0, w.num_kv_heads, w.head_size)
            out.append(np.zeros(shape, np.float32 if w.dtype == "f32" else np.uint16))
            continue
        c0, c1 = start // _CHUNK, (start + n - 1) // _CHUNK
        last_rows = (start + n - 1) % _CHUNK + 1
        parts = [_chunk_values(w, tag, stream, c, plan.outlier_channels,
                               _CHUNK if c < c1 else last_rows) for c in range(c0, c1 + 1)]
        x = np.concatenate(parts, axis=0) if len(parts) > 1 else parts[0]
        off = start - c0 * _CHUNK
        out.append(_store(w, x[off:off + n]))
    return out[0], out[1]


def seq_token_sources(plan: Plan) -> Dict[int, List[Tuple[int, int, int]]]:
    """For each sequence id, the list of (stream, start, n) runs that make up
    its logical token positions in order, after all setup and step requests."""
    runs: Dict[int, List[Tuple[int, int, int]]] = {}
    for op in list(plan.setup_ops) + list(plan.step_ops):
        if isinstance(op, AddOp):
            runs[op.seq] = []
        elif isinstance(op, ForkOp):
            runs[op.child] = list(runs[op.parent])
        else:
            r = runs[op.seq]
            if r and r[-1][0] == op.stream and r[-1][1] + r[-1][2] == op.start:
                s, st, k = r[-1]
                r[-1] = (s, st, k + op.n)
            else:
                r.append((op.stream, op.start, op.n))
    return runs


def kv_scales(plan: Plan) -> Tuple[np.ndarray, np.ndarray]:
    """Per-kv-head FP8 scales (k_scale, v_scale), float32 [H_kv]: about the
    largest |value| of a head over 448, so the N(0,1) values use the e4m3
    range; heads holding an x8 outlier channel get an 8x larger K scale."""
    w = plan.workload
    h = np.arange(w.num_kv_heads)
    k = (6.0 / 448.0) * (1.0 + 0.25 * (h % 3))
    if plan.outlier_channels.shape[0]:
        hot = np.isin(h, plan.outlier_channels[:, 0])
        k = np.where(hot, 8.0 * k, k)
    v = (5.0 / 448.0) * (1.0 + 0.25 * ((h + 1) % 3))
    return k.astype(np.float32), v.astype(np.float32)


def query_values(plan: Plan, step: int = 0) -> np.ndarray:
    """Query of the decode step, [B, H, D] in storage form; for a multi-token
    step, [num_query_rows, H, D] (the rows of sequence i start at
    ``plan.query_start[i]``)."""
    w = plan.workload
    r = _rng(w, _TAG_Q, step)
    n = plan.B if np.all(plan.query_lens == 1) else plan.num_query_rows
    q = r.standard_normal(size=(n, w.num_heads, w.head_size), dtype=np.float32)
    return _store(w, q)
