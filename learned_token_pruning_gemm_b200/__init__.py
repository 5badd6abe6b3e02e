"""TokenGate gated-prefill hot path for B200 (sm_100a).

The CUDA kernels live in libtokengate.so behind the C ABI of include/tg.h; the
Python side (api, pipeline) only marshals torch CUDA tensors to it. Importing
this package does not load the library; the first call does, and raises if it
is missing (there is no CPU fallback).
"""
__all__ = ["api", "pipeline", "synth", "build"]
