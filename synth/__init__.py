"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no attention arithmetic: it only draws random tensors, rounds
them to bfloat16 (or float16) and names the workload shapes.  Both the CUDA path and the
CPU oracle are fed from here, so that they see bit-identical inputs.
"""
from .inputs import (  # noqa: F401
    make_config_inputs,
    CONFIGS,
    AttnConfig,
    bf16_bits_to_f32,
    bits_to_f32,
    config_by_name,
    f16_bits_to_f32,
    f32_to_bf16_bits,
    f32_to_f16_bits,
    make_inputs,
    packed_lengths,
    sample_rows,
)
