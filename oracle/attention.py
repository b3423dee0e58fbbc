"""ctypes front end for the float64 C oracle of paged attention (test
infrastructure only; see the package docstring).

The C source ``attention.c`` is compiled here with gcc into
``liboracle.so`` beside it (rebuilt when the source is newer).
"""

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_ELT = {torch.float64: 0, torch.float32: 1, torch.bfloat16: 2}
_ERR = {1: "invalid batch description", 2: "block id outside the pool", 3: "out of host memory"}


def build():
    """Compile attention.c into liboracle.so (gcc -O2 -fopenmp)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            build()
        lib = ctypes.CDLL(_LIB)
        p, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_paged_attention.argtypes = [p, i32, p, p, i32, p, i32, p, p, i32, i32, i32,
                                               i32, i32, i32, i32, f64, p]
        lib.oracle_paged_attention.restype = i32
        lib.oracle_paged_attention_rows.argtypes = [p, i32, p, p, i32, p, i32, p, p, i32, i32,
                                                    i32, i32, i32, i32, i32, f64, p, i64, p]
        lib.oracle_paged_attention_rows.restype = i32
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = i32
        _lib = lib
        return lib


def num_threads():
    """Host threads one oracle call uses (OpenMP; OMP_NUM_THREADS applies)."""
    return _load().oracle_num_threads()


def set_num_threads(n):
    """Host threads for the oracle calls that follow (OpenMP's own setting, in
    the library the oracle links; the arithmetic is the same at any count)."""
    _load()
    ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))


def _cpu(t, dtype=None):
    t = t.detach().to("cpu")
    if dtype is not None:
        t = t.to(dtype)
    return t.contiguous()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _prep(q, k_pool, v_pool, block_tables, context_lens, query_start_lens):
    if q.dtype not in _ELT or k_pool.dtype not in _ELT or v_pool.dtype != k_pool.dtype:
        raise TypeError("oracle reads float64, float32 or bfloat16 tensors")
    q = _cpu(q)
    k_pool, v_pool = _cpu(k_pool), _cpu(v_pool)
    bt = _cpu(block_tables, torch.int32)
    ctx = _cpu(context_lens, torch.int32)
    qsl = _cpu(query_start_lens, torch.int32)
    if bt.dim() != 2 or q.dim() != 3 or k_pool.dim() != 4 or k_pool.shape != v_pool.shape:
        raise ValueError("expected q [T,Hq,d], pools [N,Hkv,bs,d], block_tables [B,max_blocks]")
    return q, k_pool, v_pool, bt, ctx, qsl


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, query_start_lens, scale):
    """Float64 paged attention for every query row.

    q: [num_tokens, n_q_heads, head_dim]; k_pool, v_pool: [num_blocks,
    n_kv_heads, block_size, head_dim]; block_tables: [num_seqs, max_blocks];
    context_lens: [num_seqs]; query_start_lens: [num_seqs + 1].
    Returns a float64 torch tensor shaped like q.
    """
    q, k_pool, v_pool, bt, ctx, qsl = _prep(q, k_pool, v_pool, block_tables, context_lens,
                                            query_start_lens)
    T, Hq, d = q.shape
    N, Hkv, bs, d2 = k_pool.shape
    assert d == d2
    out = torch.empty((T, Hq, d), dtype=torch.float64)
    rc = _load().oracle_paged_attention(
        _ptr(q), _ELT[q.dtype], _ptr(k_pool), _ptr(v_pool), _ELT[k_pool.dtype], _ptr(bt),
        bt.shape[1], _ptr(ctx), _ptr(qsl), ctx.shape[0], T, Hq, Hkv, d, bs, N, float(scale),
        _ptr(out))
    if rc != 0:
        raise ValueError("oracle: " + _ERR.get(rc, str(rc)))
    return out


def paged_attention_rows(q, k_pool, v_pool, block_tables, context_lens, query_start_lens, scale,
                         rows):
    """Float64 paged attention for the (token, q head) pairs in ``rows``
    ([n, 2] integer array); returns [n, head_dim] float64."""
    q, k_pool, v_pool, bt, ctx, qsl = _prep(q, k_pool, v_pool, block_tables, context_lens,
                                            query_start_lens)
    rows = torch.as_tensor(np.asarray(rows, dtype=np.int32).reshape(-1, 2)).contiguous()
    T, Hq, d = q.shape
    N, Hkv, bs, _ = k_pool.shape
    out = torch.empty((rows.shape[0], d), dtype=torch.float64)
    rc = _load().oracle_paged_attention_rows(
        _ptr(q), _ELT[q.dtype], _ptr(k_pool), _ptr(v_pool), _ELT[k_pool.dtype], _ptr(bt),
        bt.shape[1], _ptr(ctx), _ptr(qsl), ctx.shape[0], T, Hq, Hkv, d, bs, N, float(scale),
        _ptr(rows), rows.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle: " + _ERR.get(rc, str(rc)))
    return out
