"""Hadamard-rotated ("ConvRot") INT8 linear layer for NVIDIA B200 (sm_100a).

The compute lives in ``libsdnq.so`` (hand-written CUDA behind a C ABI, see
``include/sdnq.h``); this package is the thin Python binding over it.
"""
