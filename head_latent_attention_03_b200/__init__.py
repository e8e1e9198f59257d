"""B200-native Multi-head Latent Attention (MLA) decode path.

The compute lives in a C-ABI shared library (csrc/, declared in include/mla.h)
built for sm_100a; `head_latent_attention_03_b200.mla` is the thin ctypes
binding over it.  Importing this package does not load the library.
"""
__all__ = ["inputs", "mla"]
