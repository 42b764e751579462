"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no rotation, quantisation, routing or GEMM).
"""

from .workloads import (  # noqa: F401
    DIT_LINEARS,
    LINEAR_CONFIGS,
    MOE_CONFIGS,
    LinearConfig,
    MoEConfig,
    linear_inputs,
    moe_inputs,
    outlier_channels,
)
