"""Spense hybrid 2:4-sparse + dense FP8 weight GEMM for NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``lib/libspense.so`` (C ABI in
``include/spense.h``); ``spense`` is its Python binding and ``build`` compiles
it. ``synth`` and ``workloads`` build seeded synthetic inputs.
"""
