"""Per-layer routed-expert step of an expert-offloading MoE engine on one B200.

The step (router, softmax/top-k, global LRU lookup of (layer, expert) slots in
HBM, miss streaming from a pinned host pool, NVFP4 SwiGLU experts, combine)
runs in hand-written sm_100a CUDA kernels behind the C ABI of
include/moe_offload.h (libmoeoffload.so, built in-tree).  ``abi`` binds that
ABI under the same names; ``runtime`` allocates device memory and streams with
PyTorch.  There is no CPU or eager fallback.
"""
from . import abi  # noqa: F401
from .build import build  # noqa: F401

__all__ = ["abi", "build"]
