"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package holds no step of the attention method: it only draws the random
tensors (Q, K, V, page tables, sequence lengths) that both sides consume.
"""

from .workloads import WORKLOADS, Workload, Inputs, generate, get_workload  # noqa: F401
