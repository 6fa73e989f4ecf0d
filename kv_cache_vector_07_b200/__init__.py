"""libtqkv: TurboQuant compressed KV cache on one B200 (sm_100a).

The CUDA library is ``libtqkv.so`` (C ABI in ``include/tqkv.h``); the binding
lives in ``kv_cache_vector_07_b200.tqkv``.  Importing the binding fails
loudly when the library is not built.
"""
__all__ = ["tqkv", "synth", "build"]
