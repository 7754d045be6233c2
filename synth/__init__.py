"""Seeded synthetic inputs for DSA decode.

This package only draws random tensors and lays them out (CSR offsets, paged
pools, permuted page tables).  It holds none of the attention arithmetic: the
CPU oracle and the CUDA library both consume the bytes it produces.
"""
from .workloads import WORKLOADS, Workload, get_workload
from .generate import DSAInputs, make_inputs

__all__ = ["WORKLOADS", "Workload", "get_workload", "DSAInputs", "make_inputs"]
