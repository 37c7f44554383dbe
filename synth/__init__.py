"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This package only draws random numbers and names layer shapes. It holds none of
the method's arithmetic, so both the CPU oracle's tests and the CUDA library's
tests and benchmark can take their inputs from it without sharing any of the
computation under test.
"""

from .workloads import (  # noqa: F401
    LayerCase,
    LayerInputs,
    CONFIGS,
    config_cases,
    make_layer_inputs,
    make_fp4_grid_inputs,
    make_int4_grid_inputs,
    make_lora_factors,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
)
