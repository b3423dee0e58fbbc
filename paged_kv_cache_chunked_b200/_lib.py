"""ctypes loader for libpagedkv.so (argument marshalling only).

The library is built in-tree by ``paged_kv_cache_chunked_b200.build``.  A
missing library is an error: there is no fallback path.
"""

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedkv.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "paged_kv.h")

PK_OK = 0
ERRORS = {1: "PK_ERR_INVALID_ARG", 2: "PK_ERR_OOM", 3: "PK_ERR_UNSUPPORTED", 4: "PK_ERR_CUDA",
          5: "PK_ERR_BAD_INDEX", 6: "PK_ERR_WORKSPACE", 7: "PK_ERR_TIMEOUT"}
PK_F32, PK_BF16 = 0, 1
PK_ERR_TIMEOUT = 7
PK_PATH_TENSOR_CORE, PK_PATH_DECODE_BLOCKS, PK_PATH_CHUNK_TCGEN05 = 1, 2, 4


class PagedKVError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


class OutOfBlocks(PagedKVError):
    """The block manager cannot supply the blocks a call needs (state unchanged)."""


class BmStats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int64), ("free_blocks", ctypes.c_int64),
                ("used_blocks", ctypes.c_int64), ("alloc_failures", ctypes.c_int64),
                ("tail_waste_slots", ctypes.c_int64), ("num_seqs", ctypes.c_int64),
                ("host_blocks", ctypes.c_int64), ("host_free_blocks", ctypes.c_int64),
                ("prefix_lookups", ctypes.c_int64), ("prefix_hits", ctypes.c_int64),
                ("cached_blocks", ctypes.c_int64), ("state_slots", ctypes.c_int64),
                ("state_free_slots", ctypes.c_int64)]


_lib = None

_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_PP = ctypes.POINTER(ctypes.c_void_p)
_PI = ctypes.POINTER(ctypes.c_int)
_PI64 = ctypes.POINTER(ctypes.c_int64)
_PSZ = ctypes.POINTER(ctypes.c_size_t)

SIGNATURES = {
    "pk_last_error": ([], ctypes.c_char_p),
    "pk_version": ([], ctypes.c_char_p),
    "pk_pool_create": ([_I, _I, _I, _I, _I, _P, _P, _PP], _I),
    "pk_pool_destroy": ([_P], _I),
    "pk_pool_paths": ([_P, _PI], _I),
    "pk_check_device_errors": ([_P, _P, _PI], _I),
    "pk_paged_kv_append": ([_P, _P, _P, _P, _I, _P], _I),
    "pk_block_copy": ([_P, _P, _I, _P], _I),
    "pk_swap_blocks": ([_P, _P, _P, _I, _P, _I, _I, _P], _I),
    "pk_attention_workspace_size": ([_P, _I, _I, _I, _I, _PSZ], _I),
    "pk_paged_attention": ([_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P, _SZ, _P], _I),
    "pk_paged_attention_append": ([_P, _P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P, _SZ, _P], _I),
    "pk_paged_attention_noalloc": ([_P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _F, _P], _I),
    "pk_bm_create": ([_I, _I, _PP], _I),
    "pk_bm_destroy": ([_P], _I),
    "pk_bm_add_seq": ([_P, _PI64], _I),
    "pk_bm_append_slots": ([_P, _I64, _I, _P, _P, _I, _PI], _I),
    "pk_bm_blocks_needed": ([_P, _I64, _I, _PI], _I),
    "pk_bm_fork": ([_P, _I64, _PI64], _I),
    "pk_bm_free": ([_P, _I64], _I),
    "pk_bm_block_table": ([_P, _I64, _P, _I, _PI], _I),
    "pk_bm_fill_tables": ([_P, _P, _I, _P, _I], _I),
    "pk_bm_seq_len": ([_P, _I64, _PI64], _I),
    "pk_bm_refcount": ([_P, ctypes.c_int32, _PI], _I),
    "pk_bm_set_host_blocks": ([_P, _I], _I),
    "pk_bm_swap_out": ([_P, _I64, _P, _I, _PI], _I),
    "pk_bm_swap_in": ([_P, _I64, _P, _I, _PI], _I),
    "pk_bm_is_swapped": ([_P, _I64, _PI], _I),
    "pk_bm_cache_blocks": ([_P, _I64, _P, _I], _I),
    "pk_bm_cached_prefix": ([_P, _P, _I, _PI], _I),
    "pk_bm_add_seq_cached": ([_P, _P, _I, ctypes.POINTER(ctypes.c_int64), _PI], _I),
    "pk_bm_set_state_slots": ([_P, _I], _I),
    "pk_bm_state_slot": ([_P, _I64, _PI], _I),
    "pk_bm_get_stats": ([_P, ctypes.POINTER(BmStats)], _I),
    "pk_bm_num_free": ([_P, _PI], _I),
    "pk_bm_append_one_each": ([_P, _P, _I, _P, _P, _PI, _PI], _I),
}


def header_symbols():
    """Every function the public header declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(pk_[a-z0-9_]+)\s*\(", text)))


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m paged_kv_cache_chunked_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def check(rc):
    if rc != PK_OK:
        msg = lib().pk_last_error().decode(errors="replace")
        if rc == 2:
            raise OutOfBlocks(rc, msg)
        raise PagedKVError(rc, msg)
