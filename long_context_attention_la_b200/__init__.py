"""Lightning Attention layer kernel for NVIDIA B200 (sm_100a).

Submodules: ``la`` — the ctypes binding of the C ABI in include/la.h (libla_b200.so, built
in-tree by ``python -m long_context_attention_la_b200.build``); ``synth`` — seeded synthetic
inputs; ``build`` — the nvcc build.
"""
