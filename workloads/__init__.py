"""Seeded synthetic inputs for the paged KV cache hot path.

This package is the ONE thing the CUDA path and the CPU oracle share. It only
draws random numbers and lays out shapes (block tables, prior cache contents,
new-token q/k/v, norm weights); it performs none of the method's arithmetic
(no normalisation, no rotation, no rounding conversion, no attention).
"""

from .gen import (  # noqa: F401
    Workload,
    Spec,
    Segment,
    SPECS,
    make_workload,
    spec_by_name,
    NAN16,
    NAN_BITS,
    POOL_NP,
)
