"""Seeded synthetic inputs for the INT8 KV-cache workloads.

This module is shared by the CPU oracle tests and the CUDA tests / bench.
It draws random numbers and lays out shapes only; it holds none of the
quantisation or attention arithmetic.
"""
from .workloads import (  # noqa: F401
    WORKLOADS,
    EXTRA_WORKLOADS,
    ALL_WORKLOADS,
    Workload,
    bf16_normal,
    lengths_uniform,
    outlier_channels,
    apply_outliers,
    page_table_for,
    num_pages_for,
    make_decode_inputs,
)
