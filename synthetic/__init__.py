"""Seeded synthetic attention inputs with planted vertical-slash structure.

This package holds only input generation (random numbers and planted
components). It contains none of the method's arithmetic, so both the CPU
oracle and the CUDA path can consume its tensors.
"""
from .planted import Workload, WORKLOADS, make_qkv, sweep_workload, head_kinds

__all__ = ["Workload", "WORKLOADS", "make_qkv", "sweep_workload", "head_kinds"]
