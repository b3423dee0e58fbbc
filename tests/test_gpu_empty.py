"""Empty inputs through the C ABI: zero tokens to append, zero copy or swap
pairs, an attention call over zero sequences.  Each returns PK_OK, queues no
work on its stream (counted by recording the stream's work instead of running
it) and leaves the pool as it was.  The no-allocation attention call gets the
same check in tests/test_zz_no_alloc.py."""

import ctypes

import pytest
import torch

from paged_kv_cache_chunked_b200 import api
from paged_kv_cache_chunked_b200._lib import lib

from helpers import recorded_ops

pytestmark = pytest.mark.gpu

NULL = ctypes.c_void_p(0)


def _pool(dev, dtype=torch.bfloat16, d=128):
    pool = api.kv_pool_create(32, 16, 8, d, dtype, dev)
    g = torch.Generator(device="cpu").manual_seed(3)
    pool.k_pool.copy_(torch.randn(pool.k_pool.shape, generator=g).to(dtype))
    pool.v_pool.copy_(torch.randn(pool.v_pool.shape, generator=g).to(dtype))
    torch.cuda.synchronize(dev)
    return pool, pool.k_pool.clone(), pool.v_pool.clone()


def _unchanged(pool, k0, v0):
    torch.cuda.synchronize(pool.device)
    assert torch.equal(pool.k_pool, k0) and torch.equal(pool.v_pool, v0)
    assert pool.check_device_errors() == 0


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_empty_append_copy_swap(cuda_dev, dtype, d):
    torch.cuda.set_device(cuda_dev)
    pool, k0, v0 = _pool(cuda_dev, dtype, d)
    h = pool.handle
    assert recorded_ops(cuda_dev, lambda s: lib().pk_paged_kv_append(h, NULL, NULL, NULL, 0, s)) == (0, 0)
    assert recorded_ops(cuda_dev, lambda s: lib().pk_block_copy(h, NULL, 0, s)) == (0, 0)
    host = api.host_pool_create(4, pool)
    for to_host in (1, 0):
        assert recorded_ops(cuda_dev, lambda s: lib().pk_swap_blocks(
            h, ctypes.c_void_p(host.k.data_ptr()), ctypes.c_void_p(host.v.data_ptr()), 4, NULL, 0,
            to_host, s)) == (0, 0)
    # the Python wrappers take empty tensors the same way
    api.paged_kv_append(torch.empty((0, 8, d), dtype=dtype, device=cuda_dev),
                        torch.empty((0, 8, d), dtype=dtype, device=cuda_dev),
                        torch.empty((0,), dtype=torch.int64, device=cuda_dev), pool=pool)
    api.block_copy(torch.empty((0, 2), dtype=torch.int32, device=cuda_dev), pool=pool)
    _unchanged(pool, k0, v0)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_attention_over_zero_sequences(cuda_dev, dtype, d):
    torch.cuda.set_device(cuda_dev)
    pool, k0, v0 = _pool(cuda_dev, dtype, d)
    out = torch.full((4, 32, d), float("nan"), dtype=dtype, device=cuda_dev)
    qsl = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)

    def call(s):
        return lib().pk_paged_attention(pool.handle, NULL, ctypes.c_void_p(out.data_ptr()), NULL, 1,
                                        NULL, ctypes.c_void_p(qsl.data_ptr()), 0, 0, 32,
                                        ctypes.c_float(0.1), ctypes.c_void_p(ws.data_ptr()), 256, s)
    assert recorded_ops(cuda_dev, call) == (0, 0)

    def call_append(s):   # the one-call step: no rows to store, nothing to attend
        return lib().pk_paged_attention_append(pool.handle, NULL, NULL, NULL, ctypes.c_void_p(out.data_ptr()),
                                               NULL, 1, NULL, ctypes.c_void_p(qsl.data_ptr()), 0, 0, 32,
                                               ctypes.c_float(0.1), ctypes.c_void_p(ws.data_ptr()), 256, s)
    assert recorded_ops(cuda_dev, call_append) == (0, 0)
    got = api.paged_attention(torch.empty((0, 32, d), dtype=dtype, device=cuda_dev), pool.k_pool,
                              pool.v_pool, torch.empty((0, 1), dtype=torch.int32, device=cuda_dev),
                              torch.empty((0,), dtype=torch.int32, device=cuda_dev), qsl, 0.1)
    assert got.shape == (0, 32, d)
    empty_kv = torch.empty((0, 8, d), dtype=dtype, device=cuda_dev)
    got = api.paged_attention_append(torch.empty((0, 32, d), dtype=dtype, device=cuda_dev), empty_kv,
                                     empty_kv, pool.k_pool, pool.v_pool,
                                     torch.empty((0, 1), dtype=torch.int32, device=cuda_dev),
                                     torch.empty((0,), dtype=torch.int32, device=cuda_dev), qsl, 0.1)
    assert got.shape == (0, 32, d)
    assert torch.isnan(out.float()).all()
    _unchanged(pool, k0, v0)
