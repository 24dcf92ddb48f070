"""Bit-plane quantized linear layers on NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``libbq.so`` (C ABI: include/bq.h);
``bq`` is its ctypes binding. Importing this package does not load the
library; ``from bit_weight_quantization_b200 import bq`` does, and raises if
it has not been built (``python -m bit_weight_quantization_b200.build``).
"""
