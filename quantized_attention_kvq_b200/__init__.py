"""B200-native decode attention over a low-bit quantized KV cache.

The compute path is ``lib/libkvq.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/kvq.h``); ``native`` is a thin ctypes binding that
only marshals arguments.  There is no CPU fallback: every call fails loudly
when the library or a CUDA device is missing.
"""
__all__ = ["native", "workloads", "synth"]
