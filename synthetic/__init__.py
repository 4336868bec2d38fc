"""Seeded synthetic inputs for the SRU layer workloads.

This package only draws random numbers and rounds them to their storage type;
it holds none of the method's arithmetic.  Both the CPU oracle's tests and the
CUDA path's tests and benchmark take their inputs from here.
"""
from .sru_configs import (  # noqa: F401
    CONFIGS,
    SRUConfig,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    generate,
    lengths_to_mask,
)
