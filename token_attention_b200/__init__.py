"""token_attention_b200: Multi-Token Attention on NVIDIA B200 (sm_100a): the forward
pass of the attention core and of the layer, and the attention core's backward pass.

The compute lives in libmta.so (C-ABI, include/mta.h); this package holds the
thin ctypes binding (token_attention_b200.mta) and the seeded synthetic inputs
(token_attention_b200.synth).  Importing the package does not load the library;
the first call into token_attention_b200.mta does, and raises if it is missing.
"""
__all__ = ["synth", "mta"]
