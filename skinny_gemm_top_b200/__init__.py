"""B200-native weight-only low-bit quantized MoE expert matmul.

The compute lives in the C-ABI shared library built from ``csrc/`` (see
``include/qmoe.h``); ``skinny_gemm_top_b200.qmoe`` is its ctypes binding.
Importing the package does not load the library.
"""
