"""Seeded synthetic inputs for the compressed linear layer.

This package only draws random numbers and rounds them to the storage types
that the inputs are delivered in (fp32, fp16, bf16).  It contains none of the
method's arithmetic (no masking, no quantisation, no products), so that both
the CPU oracle and the CUDA path can take their inputs from here without
sharing any of the computation under test.
"""
from .gen import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_layer_inputs,
    make_activations,
    workload,
    stack_layer_specs,
)
