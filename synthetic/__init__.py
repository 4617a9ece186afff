"""Seeded synthetic inputs for MoE token dispatch / combine.

This package draws random numbers and packs them into the shapes of the
workloads; it holds none of the routing, layout, permute or combine
arithmetic. Both the CPU oracle's tests and the CUDA path's tests and
benchmark take their inputs from here.
"""

from .generator import (
    splitmix64,
    uniform01,
    standard_normal,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    zipf_bias,
    permutation,
)
from .workloads import Workload, WORKLOADS, get_workload, make_inputs

__all__ = [
    "splitmix64",
    "uniform01",
    "standard_normal",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "zipf_bias",
    "permutation",
    "Workload",
    "WORKLOADS",
    "get_workload",
    "make_inputs",
]
