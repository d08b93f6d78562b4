"""B200-native fused scaled-dot-product attention.

The compute path is the C-ABI library ``libfa.so`` (hand-written CUDA for
sm_100a, declared in ``include/fa.h``); ``flashattention_attention_b200.fa``
is its thin ctypes binding.  Importing this package does not load the
library; importing ``.fa`` does, and fails loudly when it is missing.
"""
__all__ = ["fa", "inputs"]
