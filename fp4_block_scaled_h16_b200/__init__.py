"""B200-native block-scaled FP4 quantization and block-scaled FP4 GEMM.

The compute path is the CUDA library ``libfp4.so`` (sm_100a) behind the C ABI
declared in ``include/fp4.h``; ``fp4_block_scaled_h16_b200.fp4`` is its thin
ctypes binding (argument marshalling only).  Importing this package does not
load the library; importing ``.fp4`` does, and raises if it is missing.
"""
