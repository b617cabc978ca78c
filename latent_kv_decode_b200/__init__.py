"""B200-native single-step Multi-Head Latent Attention decode.

The compute lives in ``libmla.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/mla.h``); :mod:`latent_kv_decode_b200.ops` is a thin
ctypes binding with the same call names. The library is loaded on first use;
if it is missing, every op raises instead of computing anything elsewhere.
"""
