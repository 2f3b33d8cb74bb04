"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the bench.

This package draws random numbers and rounds them to the storage types the
attention path consumes. It holds none of the attention arithmetic itself.
"""
from .inputs import (  # noqa: F401
    splitmix64,
    uniform01,
    normal,
    f32_to_bf16_bits,
    bf16_bits_to_f64,
    bf16_normal,
    bf16_normal_range,
    f32_normal,
    seed_for,
    TENSOR_Q,
    TENSOR_K,
    TENSOR_V,
    TENSOR_SINKS,
    make_prefill_inputs,
    make_decode_inputs,
)
