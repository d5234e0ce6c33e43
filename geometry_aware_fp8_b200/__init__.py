"""B200-native GIFT gradient codec: whitened FP8 / NVFP4 encode and decode.

The compute path is the C-ABI library ``libgift.so`` (hand-written sm_100a
CUDA kernels); ``geometry_aware_fp8_b200.ops`` is its thin ctypes binding.
Importing this package loads nothing: the library is opened on first use,
and every entry point raises if it is missing.
"""
__all__ = ["ops", "synth"]
