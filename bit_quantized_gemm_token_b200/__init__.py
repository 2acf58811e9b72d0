"""B200-native (sm_100a) 8-bit quantized linear layer.

The compute lives in the C-ABI library ``libw8.so`` (hand-written CUDA for sm_100a);
``bit_quantized_gemm_token_b200.w8`` is the thin Python binding with the same entry
point names.  Importing this package does not load the library; the binding loads it
on first use and raises if it is missing (there is no CPU fallback).
"""
__all__ = ["w8", "synth"]
