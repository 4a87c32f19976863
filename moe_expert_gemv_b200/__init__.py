"""B200-native affine-quantized GEMV and MoE-expert kernels.

The compute lives in ``libqmoe.so`` (CUDA, sm_100a) behind a C ABI declared in
``include/qmoe.h``; :mod:`moe_expert_gemv_b200.qmoe` is the thin ctypes
binding with the same entry-point names.  Importing this package does not load
the library; the first call does, and fails loudly if it is missing.
"""
__all__ = ["qmoe", "synth"]
