"""B200-native SageAttention-family quantized attention forward.

The compute path is the C-ABI library ``libsage.so`` (CUDA kernels for sm_100a)
declared in ``include/sage.h``; ``api`` is its thin Python binding (argument
marshalling only).  Importing this package does not load the library; the
first call into ``api`` does, and fails loudly if it is missing.
"""
__all__ = ["api", "inputs"]
