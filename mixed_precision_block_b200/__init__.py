"""B200-native DraftAttention2 mixed-precision block-sparse attention.

The compute path lives in ``libda2.so`` (CUDA for sm_100a, C ABI declared in
``include/da2.h``).  ``mixed_precision_block_b200.da2`` is the thin ctypes
binding with the same entry-point names; importing it loads the library and
fails loudly if it has not been built.  ``synth`` is the seeded input recipe.
"""
