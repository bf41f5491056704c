"""Packed low-bit KV cache and decode attention over it, for B200 (sm_100a).

The kernels live in libkvq.so (csrc/, C ABI in include/kvq.h); `kvq` is the ctypes
binding with the same entry-point names.
"""
from . import kvq  # noqa: F401
