"""B200-native (sm_100a) fused attention forward.

The product path is the C-ABI library ``libfa.so`` (hand-written CUDA for
sm_100a); :mod:`attention_attn_fwd_11_b200.fa` is a thin ctypes binding over
it.  Importing this package does not load the library; the first call does,
and it raises if the library is missing -- there is no CPU fallback.
"""
