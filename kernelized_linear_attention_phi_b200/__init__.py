"""Kernelized linear attention for NVIDIA B200 (sm_100a).

The compute runs in hand-written CUDA kernels behind a C ABI (include/la.h,
library ``_lib/libla_b200.so``); this package is the thin ctypes binding over
it plus the seeded input generators (``workloads``).
"""
