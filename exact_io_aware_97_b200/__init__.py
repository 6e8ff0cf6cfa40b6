"""Exact IO-aware attention (tiled forward and split-KV decode) for NVIDIA B200, sm_100a.

The computation lives in libfa.so (C ABI: include/fa.h); this package holds the CUDA
sources (csrc/), the nvcc build step (build.py) and a ctypes binding (binding.py).
"""
from .binding import (FA_BF16, FA_F32, FaError, decode, fa_decode, fa_decode_workspace_size, fa_device_sm_count,
                      fa_fwd, fa_fwd_workspace_size, fa_last_device_error, forward, load, status_string)

__all__ = ["FA_BF16", "FA_F32", "FaError", "decode", "fa_decode", "fa_decode_workspace_size", "fa_device_sm_count",
           "fa_fwd", "fa_fwd_workspace_size", "fa_last_device_error", "forward", "load", "status_string"]
