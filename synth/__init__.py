"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle's callers."""
from .moe_inputs import (WORKLOADS, Workload, MoEInputs, make_inputs,  # noqa: F401
                         round_to_bf16_bits, bf16_bits_to_f32, outlier_rows,
                         make_expert_biases, make_pre_norm_inputs, make_q8_experts)
