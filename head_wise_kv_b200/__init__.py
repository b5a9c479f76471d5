"""Mixed-head (DuoAttention retrieval / streaming) KV cache and attention for
B200 (sm_100a): a C-ABI CUDA library (libduo_kv.so, include/duo_kv.h) and a
thin Python binding.

``DuoKVCache`` owns the cache as a torch buffer and calls the library;
``_lib`` exposes the C functions one to one.  Both load libduo_kv.so on first
use and raise ImportError if it is missing (build it with
``python -m head_wise_kv_b200.build``); there is no fallback path.
"""
__all__ = ["DuoKVCache", "DuoError"]


def __getattr__(name):
    if name == "DuoKVCache":
        from .cache import DuoKVCache
        return DuoKVCache
    if name == "DuoError":
        from ._lib import DuoError
        return DuoError
    raise AttributeError(name)
