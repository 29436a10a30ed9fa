"""B200-native Multi-head Latent Attention over the compressed (latent) KV cache.

The compute path is the C-ABI library ``libmla.so`` (hand-written CUDA for
sm_100a); ``mla_latent_kv_31_b200.mla`` is a thin ctypes binding to it.
"""
