"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This package holds no attention or planning arithmetic: it only draws packed
sample lengths, anchor positions and bf16-rounded tensors.  Both the CUDA path
and the fp64 oracle consume exactly what it returns.
"""

from .workloads import (  # noqa: F401
    CONFIGS,
    Workload,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    make_workload,
    draw_lengths,
    draw_anchors_uniform,
    draw_anchors_beta,
)
