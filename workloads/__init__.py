"""Seeded synthetic inputs and the workload table for exact blockwise attention.

This package is shared by the CUDA path's tests and benchmark and by the oracle's
tests. It draws random numbers and describes shapes; it holds none of the
attention arithmetic (no scores, no softmax, no merge).
"""

from .configs import CONFIGS, Workload, attention_flops, get
from .gen import (
    attention_inputs,
    grid_merge_orders,
    randn_bf16,
    stress_rows,
    sample_rows,
)

__all__ = [
    "CONFIGS",
    "Workload",
    "attention_flops",
    "attention_inputs",
    "get",
    "grid_merge_orders",
    "randn_bf16",
    "sample_rows",
    "stress_rows",
]
