"""B200-native (sm_100a) SageAttention quantized attention forward.

The compute path is the CUDA library ``_lib/libsage.so`` (C ABI declared in
``include/sage.h``); ``quantized_attention_block_b200.sage`` is its thin
ctypes binding.  Importing this package does not load the library; the
binding loads it on first use and raises if it is missing.
"""
__all__ = ["workloads", "sage"]
