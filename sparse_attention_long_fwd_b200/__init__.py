"""B200 (sm_100a) Native Sparse Attention forward pass for long video token sequences.

    from sparse_attention_long_fwd_b200 import nsa      # C-ABI binding (loads libnsa_b200.so)
    from sparse_attention_long_fwd_b200 import inputs   # seeded synthetic workloads

Importing the package itself loads nothing; the shared library is loaded on first use.
"""
__version__ = "0.1.0"
