"""Seeded synthetic inputs for the block-sparse prefill workloads.

This package is shared by the CUDA path's tests and benchmark and by the
oracle.  It holds random-number generation, bf16 storage conversion and the
workload descriptions only; none of the attention, block-statistics,
selection or RoPE arithmetic lives here.
"""

from .generators import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_block_attention,
    make_inputs,
    make_mixture,
    make_tied,
    make_tiny,
)
