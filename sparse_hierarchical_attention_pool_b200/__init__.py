"""B200-native DashAttention forward pass (sm_100a CUDA kernels behind a C ABI).

``sparse_hierarchical_attention_pool_b200.dash_attn`` is the thin binding over
``libdash_attn.so``; it raises at first use when the library is missing.  Importing
this package loads nothing.
"""
