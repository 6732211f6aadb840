"""B200-native SpAtten-style cascade token/head pruning with progressive K/V quantization.

The compute lives in ``libspatten.so`` (hand-written sm_100a CUDA kernels behind a C ABI, declared
in include/spatten.h).  ``cascade_token_head_b200.spatten`` is the thin ctypes binding; it raises at
import if the library has not been built.  ``synth`` draws the seeded synthetic workloads.
"""
