"""B200-native low-bit-weight GEMM with fused dequantization.

The compute path lives in the C-ABI shared library built from ``csrc/``
(``libhq.so``); ``quantized_gemm_bit_b200.hq`` is its thin ctypes binding.
"""
