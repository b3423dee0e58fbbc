"""pk_paged_attention_noalloc: paged attention for callers that cannot
allocate device memory (a C host program with no caching allocator, a serving
loop that has reserved all free HBM for the KV pool).  It takes its scratch
from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against pk_paged_attention, on two calls in a row
(the second one finds the first one's leftovers in the shared array), within
the bf16 tolerance the other attention tests use.  This file is collected
last so that a failure here comes after every other test has run.
"""

import ctypes

import pytest
import torch

from paged_kv_cache_chunked_b200 import api
from paged_kv_cache_chunked_b200._lib import lib
from paged_kv_cache_chunked_b200.workloads import make_batch

from helpers import assert_close, gpu_pool_from

pytestmark = pytest.mark.gpu


def _noalloc(pool, b, dev):
    q = b["q"].to(dev)
    out = torch.full_like(q, float("nan"))
    tables = b["block_tables"].to(dev)
    ctx, qsl = b["context_lens"].to(dev), b["query_start_lens"].to(dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    rc = lib().pk_paged_attention_noalloc(
        pool.handle, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(tables.data_ptr()), tables.shape[1], ctypes.c_void_p(ctx.data_ptr()),
        ctypes.c_void_p(qsl.data_ptr()), ctx.shape[0], q.shape[0], q.shape[1],
        ctypes.c_float(b["scale"]), stream)
    torch.cuda.synchronize(dev)
    return rc, out


def test_noalloc_matches_the_workspace_entry_point(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    batches = [
        make_batch([900, 33, 4000, 257], [1, 33, 1, 64], block_size=16, n_q_heads=32,
                   n_kv_heads=8, head_dim=128, dtype=torch.bfloat16, seed=41),
        make_batch([1200, 77], [1, 1], block_size=16, n_q_heads=32, n_kv_heads=8,
                   head_dim=128, dtype=torch.bfloat16, seed=42),
    ]
    for b in batches:      # two calls in a row through the shared scratch array
        pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
        ref = api.paged_attention(b["q"].to(cuda_dev), pool.k_pool, pool.v_pool,
                                  b["block_tables"].to(cuda_dev), b["context_lens"].to(cuda_dev),
                                  b["query_start_lens"].to(cuda_dev), b["scale"])
        rc, got = _noalloc(pool, b, cuda_dev)
        assert rc == 0, lib().pk_last_error()
        assert_close(got, ref, torch.bfloat16, "no-alloc vs workspace entry point")
        assert pool.check_device_errors() == 0


def test_noalloc_refuses_batches_beyond_its_scratch(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    b = make_batch([64], [1], block_size=16, n_q_heads=32, n_kv_heads=8, head_dim=128,
                   dtype=torch.bfloat16, seed=43, poison_unused=False)
    pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
    need = ctypes.c_size_t()
    # 512 sequences with 16 q heads per kv head: split-K scratch past 32 MiB
    n_seqs, n_q_heads = 512, 128
    lib().pk_attention_workspace_size(pool.handle, n_seqs, n_seqs, n_q_heads, 4, ctypes.byref(need))
    assert need.value > 32 << 20
    dummy = ctypes.c_void_p(pool.k_pool.data_ptr())
    rc = lib().pk_paged_attention_noalloc(pool.handle, dummy, dummy, dummy, 4, dummy, dummy, n_seqs,
                                          n_seqs, n_q_heads, ctypes.c_float(1.0), None)
    assert rc == 6                             # PK_ERR_WORKSPACE, nothing launched
    assert b"scratch" in lib().pk_last_error()
