"""Seeded synthetic inputs for paged decode attention.

This package only draws sizes, orders and values; it holds no arithmetic of
the method (no block/slot mapping, no softmax, no allocator logic).  The
CPU oracle, the CUDA-path tests and the benchmark all take their inputs
from here, so that both sides of every parity check see identical data.
"""

from .synth import (  # noqa: F401
    BLOCK_SIZE,
    WORKLOADS,
    Workload,
    Plan,
    AppendOp,
    AddOp,
    ForkOp,
    make_plan,
    stream_kv,
    seq_token_sources,
    query_values,
    kv_scales,
    to_bf16_bits,
    bf16_bits_to_f32,
    workload_by_name,
)
