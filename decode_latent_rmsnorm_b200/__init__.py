"""B200-native MLA latent-KV hot path: latent RMSNorm + kv_b_proj, YaRN RoPE,
causal prefill attention and absorbed split-KV decode, in hand-written sm_100a
CUDA behind the C-ABI library ``libmla.so`` (declared in ``include/mla.h``).

``decode_latent_rmsnorm_b200.mla`` is the thin ctypes binding; the library is
loaded on first use and its absence is an error (there is no fallback).
"""
