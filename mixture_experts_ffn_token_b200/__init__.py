"""B200 (sm_100a) stacked Mixture-of-Experts FFN forward pass.

The compute lives in libmoe_b200.so (hand-written CUDA kernels behind the C
ABI of include/moe.h); `abi` is its thin ctypes binding and `workloads` the
seeded synthetic input generator.  Importing the package does not load the
library; the first call into `abi` does, and raises if it is missing.
"""
from . import workloads  # noqa: F401

__all__ = ["abi", "workloads"]
