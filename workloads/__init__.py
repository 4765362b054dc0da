"""Seeded synthetic inputs for the MoE forward pass.

This package is the one piece of code that both the CPU oracle's tests and the
CUDA path's tests/bench use.  It draws random numbers and rounds them to the
storage dtype; it contains none of the layer's arithmetic (no routing, no
softmax, no experts).  See ``generate.py``.
"""
from .generate import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_expert_weights,
    make_inputs,
    make_exact_router_inputs,
)
