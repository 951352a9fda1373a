"""B200-native per-rank compute of context-parallel (ring / Ulysses / 2D) causal attention.

The compute lives in the CUDA library ``libcpattn.so`` (C ABI, ``include/cp_attn.h``);
``binding`` marshals torch tensors into that ABI.  ``synth`` holds the seeded input
generator.  Importing this package does not load the library; the first binding call does,
and fails loudly if it is missing.
"""
