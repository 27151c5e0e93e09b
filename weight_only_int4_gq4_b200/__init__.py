"""Grouped-int4 (fmt=4, gs=64) weight-only MoE expert FFN for B200 (sm_100a).

The compute lives in ``libgq4.so`` (hand-written CUDA behind a C ABI, declared in
``include/gq4.h``).  ``weight_only_int4_gq4_b200.gq4`` is the thin Python binding over
it; importing that module loads the library and fails loudly when it is missing.
``weight_only_int4_gq4_b200.synth`` holds the seeded synthetic input generators.
"""
