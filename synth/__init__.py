"""Seeded synthetic inputs for the multi-LoRA delta path.

This package draws inputs only: activations, adapter weights, adapter ids,
segment lengths and page-scatter seeds.  It holds none of the delta's
arithmetic and is shared by the tests, the benchmark and the smoke check, so
that the CUDA path and the CPU oracle see byte-identical inputs.
"""

from .workloads import (  # noqa: F401
    Workload,
    bf16_bits_to_f32,
    config,
    custom,
    f32_to_bf16_bits,
    integer_case,
    normal_bf16,
    zipf_lengths,
)
