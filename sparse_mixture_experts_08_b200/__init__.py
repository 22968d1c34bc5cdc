"""B200-native (sm_100a) forward pass of one sparse Mixture-of-Experts layer.

The computation lives in ``libmoe.so`` (CUDA kernels behind the C ABI of
``include/moe.h``); ``moe`` is its ctypes binding.
"""
from . import moe  # noqa: F401
from .moe import *  # noqa: F401,F403
