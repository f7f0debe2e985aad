"""FP8 (E4M3) attention forward pass for B200 with a static P-cast scale.

The compute path is the hand-written sm_100a CUDA library ``libfp8attn.so``
(C ABI in ``include/fp8attn.h``); :mod:`softmax_cast_precision_b200.fp8attn`
is its Python binding.  There is no CPU or library fallback: if the library
is missing the binding raises.
"""

__all__ = ["fp8attn"]
