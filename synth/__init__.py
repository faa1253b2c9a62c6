"""Seeded synthetic decode workloads (host numpy generator + device fill library).

Shared by the oracle's tests and the CUDA path; contains none of the method's arithmetic.
"""
from .gen import (  # noqa: F401
    Needles, Workload, bf16_bits_to_f32, f64_to_bf16_bits, gen_k_rows, gen_needles, gen_q,
    gen_v_rows, host_head, host_layer, key_offset, normal_f64, pct_k, plant, raw_u64,
    stream_key, sweep_names, workload,
)
