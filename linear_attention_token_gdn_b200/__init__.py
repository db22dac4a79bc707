"""B200-native Gated DeltaNet (GDN) token mixer.

The compute lives in ``libgdn.so`` (hand-written CUDA for sm_100a behind a C ABI,
declared in ``include/gdn.h``).  ``linear_attention_token_gdn_b200.gdn`` is the thin
ctypes binding with the same entry-point names; ``.inputs`` draws the seeded
synthetic workloads; ``.build`` compiles the library in-tree.
"""
