"""B200-native FP4 (ExMy) weight quantization and W4A16 GEMM.

The compute path lives in the CUDA library ``libfp4w4a16.so`` (sources in
``csrc/``, C interface in ``include/fp4w4a16.h``); ``api`` is a thin ctypes
binding over it that uses PyTorch only for device memory and streams.
"""
