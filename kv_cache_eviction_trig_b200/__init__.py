"""B200-native (sm_100a) TriAttention KV-cache prune step.

The compute lives in ``libtria.so`` (CUDA, built from ``csrc/``) behind the C
ABI in ``include/tria.h``; ``tria`` is its ctypes binding and ``workloads``
draws the seeded synthetic caches used by the tests and the benchmark.
"""
from . import tria, workloads  # noqa: F401

__all__ = ["tria", "workloads"]
