"""B200-native W4A4 quantized linear layer (INT4 activations x INT4 weights).

The compute runs in the CUDA library ``libfq.so`` (C ABI declared in
``include/fq.h``); ``int4_linear_b200.fq`` is its thin Python binding.
"""
__all__ = ["fq", "synth"]
