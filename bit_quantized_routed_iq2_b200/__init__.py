"""Routed 2-bit MoE FFN for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libmoe2bit.so`` (C ABI in
``include/moe2bit.h``); ``moe2bit`` is its ctypes binding.
"""
from . import moe2bit  # noqa: F401
