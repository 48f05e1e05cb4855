"""Parallel-Newton evaluation of GRU recurrences on NVIDIA B200 (sm_100a).

The compute lives in ``libpararnn.so`` (CUDA kernels behind the C ABI of
``include/pararnn.h``); ``binding`` marshals torch tensors into it and
``inputs`` draws the seeded synthetic workloads.  Importing the package does
not load the library; the first call does, and raises if it is missing.
"""
from .binding import (  # noqa: F401
    SolveResult, affine_scan, alloc_workspace, newton_solve, solve_workload, workspace_size,
)
