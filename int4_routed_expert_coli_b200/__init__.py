"""B200-native routed-expert MoE layer with int4 gs64 experts.

Submodules:
  coli_moe  - ctypes binding of libcoli_moe.so (the C ABI, include/coli_moe.h)
  synth     - seeded synthetic inputs (weights, activations, logits, routing)
  build     - builds libcoli_moe.so for sm_100a
"""
