"""Seeded synthetic workloads for the CoSA prefill path.

This package holds input generation only: random tensors, the planted
attention structure of each workload, bf16 encoding and the paged KV layout.
It contains none of the method's arithmetic, so both the CPU oracle's tests
and the CUDA path can draw their inputs from it.
"""

from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    bf16_bits,
    bf16_bits_to_f32,
    from_arrays,
    make_workload,
    make_custom,
)
