"""Seeded synthetic inputs for the HISA indexer.

This package is shared by the CPU oracle tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and lays them out; it holds none of
the indexer's arithmetic (no pooling, scoring or selection).
"""

from .workloads import (  # noqa: F401
    BF16_ONE,
    Workload,
    DecodeWorkload,
    bf16_from_f32,
    bf16_to_f32,
    integer_prefill,
    gaussian_prefill,
    needle_prefill,
    varlen_prefill,
    varlen_lengths,
    decode_workload,
    config_workload,
    CONFIG_NAMES,
)
