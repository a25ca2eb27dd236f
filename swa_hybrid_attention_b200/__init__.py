"""Headwise hybrid (SWA + sparse retrieval) prefill/decode attention for B200.

The compute lives in ``librtp.so`` (hand-written CUDA for sm_100a behind a C
ABI declared in include/rtp.h); ``swa_hybrid_attention_b200.rtp`` is the thin
ctypes binding with the same function names.  ``inputs`` generates the seeded
synthetic workloads.  Submodules are imported explicitly
(``from swa_hybrid_attention_b200 import rtp``) so that input generation
works on machines without a GPU.
"""
