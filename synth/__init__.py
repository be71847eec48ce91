"""Seeded synthetic workloads for the INT8 ConvRot linear layer.

This package only draws inputs (activations, weights, bias) and stores them as
bf16 bit patterns. It holds none of the method's arithmetic: no rotation, no
quantisation, no GEMM. Both the CPU oracle's tests and the CUDA path's tests
and benchmark take their inputs from here.
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    gelu_bf16_bits,
    make_workload,
)
