"""Routed-MoE layer forward (int4/int8 expert GEMV + router) for NVIDIA B200, sm_100a.

The compute lives in the C-ABI library libmoe.so (include/moe.h); `abi` is its
ctypes binding.  Importing this package does not load the library; the first
call does, and fails loudly if it has not been built.
"""
from . import abi  # noqa: F401

__all__ = ["abi"]
