"""B200-native (sm_100a) QLoRA-linear hot path: NF4 blockwise quantization,
double quantization of the block constants, and the fused forward/backward of
y = doubleDequant(W0) x + s B (A x).

The compute lives in ``libqlora_nf4.so`` (hand-written CUDA, C ABI declared in
``include/qlora_nf4.h``); ``api`` is the thin ctypes binding over it.  Importing
this package does not load the library: ``api`` loads it on first use and
raises if it is missing.  ``synthetic`` holds the seeded workloads.
"""
__all__ = ["api", "synthetic"]
