"""Seeded synthetic inputs for the SERQ linear (activations, weights, workloads).

This module only draws random numbers and rounds them to the bf16 storage type.
It holds none of the method's arithmetic (no scaling, permutation, quantization
or products), so that both the CPU oracle and the CUDA path can be fed from it
without sharing any of the computation they are compared on.
"""

from .generators import (  # noqa: F401
    Linear,
    Workload,
    activations,
    bf16_bits,
    norm_weight,
    round_to_bf16,
    weights,
    workload,
    WORKLOADS,
)
