"""GPT-OSS Mixture-of-Experts FFN layer on B200 (sm_100a): C-ABI CUDA library + thin binding.

The compute lives in ``libmoe.so`` (csrc/, include/moe.h); ``api`` marshals torch
tensors into its calls.  Importing this package does not load the library;
the first call does, and fails loudly if it is missing.
"""
from . import _lib  # noqa: F401

__all__ = ["api", "build"]
