"""Cut Cross-Entropy for B200 (sm_100a): Python binding of libcce.so.

The binding only marshals arguments; every step of the loss and its gradient
runs in the library's CUDA kernels.  The native library is loaded on first use
and a missing or unloadable library raises immediately (there is no CPU
fallback).
"""
