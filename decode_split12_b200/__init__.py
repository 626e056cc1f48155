"""Split12: lossless 12-bit BF16 weights with fused decode-GEMV/GEMM on B200.

The compute path lives in the CUDA library ``libs12.so`` (C ABI declared in
``include/s12.h``); ``decode_split12_b200.s12`` is the thin ctypes binding.
Importing this package does not load the library; the binding does, and it
raises if the library is missing.
"""
__version__ = "0.1.0"
