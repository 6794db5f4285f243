"""Seeded synthetic inputs for the MISA indexer path.

This package holds input generators and the workload shape table only.  It
contains none of the method's arithmetic (no pooling, routing, scoring or
selection), so both the CPU oracle and the CUDA path can draw their inputs
from it without sharing any computation.
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    IndexerInputs,
    make_inputs,
    fp32_to_bf16_bits,
    sample_rows,
)
