"""liblkv for B200: group-wise asymmetric low-bit KV cache (K6V4 and 8/4/2-bit
variants) and single-token decode attention over the packed cache, with the
sparse-V skip and the attention-tiered cache.

The compute lives in liblkv.so (hand-written sm_100a CUDA behind the C ABI of
include/lkv.h); ``lkv`` is its thin ctypes binding, ``buffers`` allocates the
device tensors, ``workloads`` draws seeded synthetic inputs.
"""
from . import buffers, lkv, workloads  # noqa: F401

__all__ = ["buffers", "lkv", "workloads"]
