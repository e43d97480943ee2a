"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and the bench.

This package holds no GEMM arithmetic and no scale-factor packing: it only draws
random numbers and encodes them into the operand formats (the quantisation recipe
that produces the operands the block-scaled GEMM consumes).  Both the CUDA path and
the oracle receive the same bytes from here.
"""

from .synth import (  # noqa: F401
    QMAX_E4M3,
    QMAX_E2M1,
    ue8m0_exponent_for_amax,
    quantize_e4m3_blocks,
    quantize_e2m1_blocks,
    bf16_operand,
    normal_matrix,
    dense_fp8_problem,
    dense_fp4_problem,
    dense_bf16_problem,
    grouped_fp8_problem,
    masked_fp8_problem,
    dirichlet_segments,
)
