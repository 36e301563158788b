"""Seeded synthetic inputs for the QSA decode step.

This package only draws random numbers and lays them out (token arrays,
queries, head weights, page tables). It holds none of the method's
arithmetic: no compression, scoring, selection or attention. Both the CPU
oracle tests and the CUDA path read their inputs from here, so that the two
sides always see the same bytes.
"""

from .workloads import (  # noqa: F401
    Dims,
    Workload,
    PRESETS,
    preset_spec,
    make_workload,
    make_custom,
    step_queries,
    prefill_queries,
    seed_for,
)
