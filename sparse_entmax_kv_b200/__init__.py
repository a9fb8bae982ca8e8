"""B200-native EntmaxKV: paged, support-aware alpha-entmax decode attention.

The compute lives in libentmaxkv.so (CUDA, sm_100a; C ABI in
include/entmaxkv.h).  ``native`` is the ctypes binding, ``decoder`` strings the
calls of one decode step together, ``workloads`` draws seeded synthetic inputs.
"""
__all__ = ["native", "decoder", "workloads"]
