"""HiLS (Hierarchical Landmark Sparse) attention forward pass for NVIDIA B200.

The compute lives in ``libhils.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/hils.h``); this package only marshals arguments
to it.  See ``binding.py`` for the Python entry points.
"""
from .workloads import WORKLOADS, Workload  # noqa: F401
