"""B200-native Wan2.1 / Wan2.2 DiT block forward and CFG flow-matching Euler
step: a C-ABI CUDA library (``libwan.so``, sm_100a) and a thin ctypes binding.

The binding only marshals arguments; every step of the path runs in the
library's kernels. Importing the binding on a machine without the built
library raises (there is no CPU fallback).
"""
from . import configs  # noqa: F401

__all__ = ["configs"]
