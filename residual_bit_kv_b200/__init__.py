"""B200-native ResidualQuant KV cache: quantize-and-append of looped-Transformer
KV states and the compressed decode-attention kernel (librq).

The CUDA library is loaded lazily by :mod:`residual_bit_kv_b200.librq`;
importing the package itself loads no native code.
"""
__all__ = ["librq", "synth"]
