"""MoBA (Mixture of Block Attention) causal prefill forward pass for NVIDIA B200 (sm_100a).

The compute path lives in libmoba.so (hand-written CUDA kernels behind the C ABI of
include/moba.h); `moba` is its ctypes binding and `workloads` draws seeded synthetic inputs.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "moba"]
