"""Seeded synthetic inputs shared by the oracle side and the GPU side.

This package holds no attention arithmetic.  It draws the random tensors of
the reference workloads (shapes, value distributions and structure taken from
the attention pages), rounds them to the storage dtype, and hands the same
bits to both the float64 oracle and the CUDA library.
"""

from .workloads import (  # noqa: F401
    RECIPES,
    Recipe,
    bf16_bits_to_f64,
    bf16_round_bits,
    generate,
    normal_f64,
    stream_key,
    tensor_slice_f64,
    uniform_f64,
)
