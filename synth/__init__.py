"""Seeded synthetic inputs for SAS gated block-sparse attention.

This package only draws random numbers and rounds them to bf16. It holds none
of the attention arithmetic, so both the fp64 oracle and the CUDA path can take
their inputs from it without sharing any of the method's code.
"""
from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    bf16_round,
    bf16_bits,
    bits_to_f32,
    prefill_inputs,
    decode_inputs,
    sweep_workloads,
)
