"""Seeded synthetic inputs for the SketchSSM windowed-decode workloads.

This package draws random numbers and shapes them into the per-token inputs
(q, k, v, decay, beta) and the calibration queries of the Mamba-2, Gated
DeltaNet and KDA decode workloads.  It holds none of the method's arithmetic:
no recurrence, no read, no sketch, no calibration.  Both the CPU oracle and the
CUDA path take their inputs from here, and neither is imported by this package.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    KINDS,
    Workload,
    calibration_queries,
    query_basis,
    sample_heads,
    token_block,
    workload,
)
