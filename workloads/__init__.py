"""Seeded synthetic workloads for the paged decode path.

This package only draws random inputs and lays them out; it holds none of the
method's arithmetic (no attention, no slot computation, no block accounting),
so both the CUDA path and the oracle can be fed from it.
"""
from .synth import (  # noqa: F401
    CONFIGS,
    Workload,
    fill_normal_fp16,
    make_workload,
    normal_fp16,
    random_distinct_slots,
)
