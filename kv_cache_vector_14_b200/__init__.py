"""TurboQuant KV-cache compression and compressed-cache decode attention for
NVIDIA B200 (sm_100a).

The compute lives in ``libtq.so`` (CUDA kernels behind the C ABI declared in
``include/tq.h``); ``kv_cache_vector_14_b200.tq`` is the thin ctypes binding.
Importing the package itself loads nothing, so ``synthetic`` (input
generators) can be used without a GPU.
"""
__all__ = ["tq", "synthetic"]
