"""Test helpers: put a seeded workload on the GPU through the library's own
entry points, and compare with the oracle.

Device side (the product path): the C++ allocator turns each request into
slots and copy-on-write pairs; per serving step the pairs go through
pa_copy_blocks and then the step's tokens through pa_reshape_and_cache.
Host side: oracle.replay applies the same requests one by one.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np
import torch

import paged_kv_cache_351_b200 as pa
from oracle.attention import widen
from workloads import AddOp, AppendOp, ForkOp, Plan, kv_scales, query_values, stream_kv

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}
TOL = {"f32": 1e-5, "bf16": 1e-2}


def to_device_values(raw: np.ndarray, dtype: str, device) -> torch.Tensor:
    """Storage-form numpy (float32 or bf16 bits) -> torch tensor of that dtype."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(raw)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).to(device)
    return t.view(torch.bfloat16)


def to_host_raw(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "f32":
        return t.numpy()
    if dtype == "fp8":
        return t.view(torch.uint8).numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


@dataclass
class DeviceState:
    plan: Plan
    alloc: pa.Allocator
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_tables: torch.Tensor  # int32 [B, max_nb] on device
    context_lens: torch.Tensor  # int32 [B] on device
    tables_host: np.ndarray
    lens_host: np.ndarray
    cow_pairs: List[tuple]
    step_slots: Optional[torch.Tensor] = None  # int64 [B] device: slots of the step's new tokens
    step_key: Optional[torch.Tensor] = None
    step_value: Optional[torch.Tensor] = None
    k_scale: Optional[torch.Tensor] = None  # FP8 cache only
    v_scale: Optional[torch.Tensor] = None

    def write(self, key, value, slots):
        if self.k_scale is not None:
            pa.pa_reshape_and_cache_fp8(key, value, self.k_cache, self.v_cache, slots, self.k_scale, self.v_scale)
        else:
            pa.pa_reshape_and_cache(key, value, self.k_cache, self.v_cache, slots)


def build_device_state(plan: Plan, device="cuda", include_step=True, write_step=True,
                       stop_after: Optional[int] = None) -> DeviceState:
    w = plan.workload
    dt = TORCH_DTYPE[w.cache_dtype]
    shape = (plan.num_blocks, w.num_kv_heads, w.block_size, w.head_size)
    k_cache = torch.empty(shape, dtype=dt, device=device)
    v_cache = torch.empty(shape, dtype=dt, device=device)
    ks = vs = None
    if w.cache_dtype == "fp8":
        ks_np, vs_np = kv_scales(plan)
        ks, vs = torch.from_numpy(ks_np).to(device), torch.from_numpy(vs_np).to(device)
    alloc = pa.Allocator(plan.num_blocks, w.block_size, plan.free_order)
    cow_all: List[tuple] = []

    pend_slots: List[np.ndarray] = []
    pend_k: List[np.ndarray] = []
    pend_v: List[np.ndarray] = []
    pend_pairs: List[tuple] = []
    pend_seqs = set()

    def flush():
        if pend_pairs:
            pairs = torch.tensor(pend_pairs, dtype=torch.int64, device=device)
            pa.pa_copy_blocks(k_cache, v_cache, pairs)
        if pend_slots:
            slots = torch.from_numpy(np.concatenate(pend_slots)).to(device)
            key = to_device_values(np.concatenate(pend_k), w.dtype, device)
            value = to_device_values(np.concatenate(pend_v), w.dtype, device)
            if ks is not None:
                pa.pa_reshape_and_cache_fp8(key, value, k_cache, v_cache, slots, ks, vs)
            else:
                pa.pa_reshape_and_cache(key, value, k_cache, v_cache, slots)
        pend_slots.clear(), pend_k.clear(), pend_v.clear(), pend_pairs.clear(), pend_seqs.clear()

    ops = list(plan.setup_ops) + (list(plan.step_ops) if include_step else [])
    if stop_after is not None:
        ops = ops[:stop_after]
    n_setup = len(plan.setup_ops)
    step_slots = []
    for idx, op in enumerate(ops):
        if isinstance(op, AddOp):
            alloc.add(op.seq)  # a new sequence touches no pending block
        elif isinstance(op, ForkOp):
            flush()
            alloc.fork(op.parent, op.child)
        else:
            if op.seq in pend_seqs:  # a new serving step begins
                flush()
            slots, cow = alloc.append(op.seq, op.n)
            cow_all += cow
            if idx >= n_setup:
                step_slots.append(slots)
                if not write_step:
                    continue
            k, v = stream_kv(plan, op.stream, op.start, op.n)
            pend_slots.append(slots)
            pend_k.append(k)
            pend_v.append(v)
            pend_pairs.extend(cow)
            pend_seqs.add(op.seq)
            if sum(len(s) for s in pend_slots) > 200_000:
                flush()
    flush()
    max_nb = plan.max_blocks_per_seq
    tables, lens = alloc.block_tables(plan.batch, max_nb)
    st = DeviceState(plan, alloc, k_cache, v_cache, torch.from_numpy(tables).to(device),
                     torch.from_numpy(lens).to(device), tables, lens, cow_all, k_scale=ks, v_scale=vs)
    if include_step and plan.step_ops:
        st.step_slots = torch.from_numpy(np.concatenate(step_slots)).to(device)
        ks, vs = [], []
        for op in plan.step_ops:
            k, v = stream_kv(plan, op.stream, op.start, op.n)
            ks.append(k)
            vs.append(v)
        st.step_key = to_device_values(np.concatenate(ks), w.dtype, device)
        st.step_value = to_device_values(np.concatenate(vs), w.dtype, device)
    torch.cuda.synchronize()
    return st


def decode_on_device(st: DeviceState, query: torch.Tensor, partition_tokens: int = 0,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    w = st.plan.workload
    if out is None:
        out = torch.empty_like(query)
    n = pa.pa_decode_workspace_bytes(st.plan.B, w.num_heads, w.num_kv_heads, w.head_size,
                                     st.block_tables.shape[1], partition_tokens)
    ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=query.device) if n else None
    if st.k_scale is not None:
        pa.pa_decode_fp8(out, query, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                         1.0 / np.sqrt(w.head_size), w.num_kv_heads, st.k_scale, st.v_scale, workspace=ws,
                         partition_tokens=partition_tokens)
    else:
        pa.pa_decode(out, query, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                     1.0 / np.sqrt(w.head_size), w.num_kv_heads, workspace=ws, partition_tokens=partition_tokens)
    return out


def device_query(plan: Plan, device="cuda", step: int = 0) -> torch.Tensor:
    return to_device_values(query_values(plan, step), plan.workload.dtype, device)


def max_abs_err(gpu_out: torch.Tensor, ref: Dict[int, np.ndarray], dtype: str) -> float:
    got = widen(to_host_raw(gpu_out, dtype), dtype)
    return max(float(np.max(np.abs(got[i] - r))) if r.size else 0.0 for i, r in ref.items())


def check_status_clean():
    st, bits = pa.pa_get_device_status()
    assert st == 0 and bits == 0, f"device status {st} bits {bits:#x}"
