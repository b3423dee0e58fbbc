"""Paged KV cache with chunked prefill for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libpagedkv.so`` (hand-written CUDA
kernels); this package is its thin Python binding plus the host-side
scheduler.  Importing the package does not load the library; the first call
that needs it does, and fails loudly if it has not been built.
"""

__all__ = ["kv_pool_create", "paged_kv_append", "paged_attention", "block_copy",
           "BlockManager", "KVPool"]


def __getattr__(name):
    if name in __all__:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
