"""GPU parity of the two copy kernels against the oracle: bit-exact.

Append ["PagedAttention & Continuous Batching" (study notes), "Flow" step 4]
and whole-block copy for copy-on-write [same page, "Copy-on-write"], through
the C ABI, on pools whose other contents must stay untouched (canaries)."""

import pytest
import torch

import oracle
from paged_kv_cache_chunked_b200 import api

pytestmark = pytest.mark.gpu

GEOMS = [
    # num_blocks, block_size, Hkv, d, dtype
    (64, 16, 8, 128, torch.bfloat16),
    (40, 8, 4, 256, torch.bfloat16),
    (33, 32, 2, 64, torch.float32),
    (20, 4, 3, 40, torch.bfloat16),   # 80-byte rows: element-wise kernel
    (17, 1, 1, 5, torch.float32),     # 20-byte rows: element-wise kernel
]


def _random_pool(pool, seed):
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(pool.k_pool.shape, generator=g).to(pool.dtype)
    vc = torch.randn(pool.v_pool.shape, generator=g).to(pool.dtype)
    pool.k_pool.copy_(kc)
    pool.v_pool.copy_(vc)
    return kc, vc


@pytest.mark.parametrize("geom", GEOMS)
def test_append_bit_exact(cuda_dev, geom):
    N, bs, Hkv, d, dtype = geom
    pool = api.kv_pool_create(N, bs, Hkv, d, dtype, cuda_dev)
    kc, vc = _random_pool(pool, 1)
    g = torch.Generator().manual_seed(2)
    T = min(N * bs, 3 * bs + 5)
    slots = torch.randperm(N * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1                                   # skipped tokens
    k = torch.randn((T, Hkv, d), generator=g).to(dtype)
    v = torch.randn((T, Hkv, d), generator=g).to(dtype)
    api.paged_kv_append(k.to(cuda_dev), v.to(cuda_dev), slots.to(cuda_dev), pool=pool)
    oracle.kv_append(kc, vc, k, v, slots)
    torch.cuda.synchronize()
    assert torch.equal(pool.k_pool.cpu(), kc)
    assert torch.equal(pool.v_pool.cpu(), vc)
    assert pool.check_device_errors() == 0


def test_append_large_batch_bit_exact(cuda_dev):
    # a 512-token prefill chunk for each of 64 sequences into a shuffled pool
    N, bs, Hkv, d = 4096, 16, 8, 128
    pool = api.kv_pool_create(N, bs, Hkv, d, torch.bfloat16, cuda_dev)
    g = torch.Generator(device=cuda_dev).manual_seed(3)
    T = 64 * 512
    slots = torch.randperm(N * bs, generator=g, device=cuda_dev)[:T]
    k = torch.randn((T, Hkv, d), generator=g, device=cuda_dev).to(torch.bfloat16)
    v = torch.randn((T, Hkv, d), generator=g, device=cuda_dev).to(torch.bfloat16)
    api.paged_kv_append(k, v, slots, pool=pool)
    torch.cuda.synchronize()
    s = slots.cpu()
    blk, off = s // bs, s % bs
    # every token's rows, all heads, landed where its slot points
    assert torch.equal(pool.k_pool[blk.to(cuda_dev), :, off.to(cuda_dev)].cpu(), k.cpu())
    assert torch.equal(pool.v_pool[blk.to(cuda_dev), :, off.to(cuda_dev)].cpu(), v.cpu())


def test_append_rejects_out_of_range_slot_without_writing(cuda_dev):
    pool = api.kv_pool_create(4, 4, 1, 8, torch.float32, cuda_dev)
    k = torch.ones((2, 1, 8), device=cuda_dev)
    slots = torch.tensor([3, 16], dtype=torch.int64, device=cuda_dev)   # 16 is past the pool
    api.paged_kv_append(k, k, slots, pool=pool)
    torch.cuda.synchronize()
    assert pool.check_device_errors() == 5      # PK_ERR_BAD_INDEX recorded
    assert float(pool.k_pool.sum()) == 8.0       # only slot 3 written
    assert pool.check_device_errors() == 0      # the check clears the word


@pytest.mark.parametrize("geom", GEOMS)
def test_block_copy_bit_exact(cuda_dev, geom):
    N, bs, Hkv, d, dtype = geom
    pool = api.kv_pool_create(N, bs, Hkv, d, dtype, cuda_dev)
    kc, vc = _random_pool(pool, 5)
    g = torch.Generator().manual_seed(6)
    perm = torch.randperm(N, generator=g)
    n = N // 3
    pairs = torch.stack([perm[:n], perm[n:2 * n]], 1).to(torch.int32)   # dsts distinct, not srcs
    api.block_copy(pairs.to(cuda_dev), pool=pool)
    oracle.block_copy(kc, vc, pairs)
    torch.cuda.synchronize()
    assert torch.equal(pool.k_pool.cpu(), kc)
    assert torch.equal(pool.v_pool.cpu(), vc)
    assert pool.check_device_errors() == 0


def test_block_copy_many_pairs(cuda_dev):
    N = 8192
    pool = api.kv_pool_create(N, 16, 8, 128, torch.bfloat16, cuda_dev)
    g = torch.Generator(device=cuda_dev).manual_seed(7)
    pool.k_pool.copy_(torch.randn(pool.k_pool.shape, generator=g, device=cuda_dev))
    pool.v_pool.copy_(torch.randn(pool.v_pool.shape, generator=g, device=cuda_dev))
    perm = torch.randperm(N, generator=g, device=cuda_dev).to(torch.int32)
    pairs = torch.stack([perm[:4096], perm[4096:]], 1).contiguous()
    k0, v0 = pool.k_pool.clone(), pool.v_pool.clone()
    api.block_copy(pairs, pool=pool)
    torch.cuda.synchronize()
    src, dst = pairs[:, 0].long(), pairs[:, 1].long()
    assert torch.equal(pool.k_pool[dst], k0[src]) and torch.equal(pool.v_pool[dst], v0[src])
    assert torch.equal(pool.k_pool[src], k0[src])


@pytest.mark.parametrize("geom", GEOMS)
def test_swap_blocks_round_trip_bit_exact(cuda_dev, geom):
    # swap-out to a pinned host pool and swap-in to other device blocks
    # ["Batching and PagedAttention", "When blocks run out"], against the
    # oracle's whole-block moves; untouched blocks on both sides stay as they were
    N, bs, Hkv, d, dtype = geom
    pool = api.kv_pool_create(N, bs, Hkv, d, dtype, cuda_dev)
    kc, vc = _random_pool(pool, 11)
    H = N // 2 + 1
    host = api.host_pool_create(H, pool)
    g = torch.Generator().manual_seed(12)
    host.k.copy_(torch.randn(host.k.shape, generator=g).to(dtype))
    host.v.copy_(torch.randn(host.v.shape, generator=g).to(dtype))
    hk, hv = host.k.clone(), host.v.clone()
    n = min(N // 3, H)
    out_pairs = torch.stack([torch.randperm(N, generator=g)[:n], torch.randperm(H, generator=g)[:n]], 1)
    out_pairs = out_pairs.to(torch.int32)
    api.swap_blocks(out_pairs.to(cuda_dev), to_host=True, host_pool=host, pool=pool)
    oracle.swap_blocks(kc, vc, hk, hv, out_pairs, to_host=True)
    torch.cuda.synchronize()
    assert torch.equal(host.k, hk) and torch.equal(host.v, hv)
    in_pairs = torch.stack([out_pairs[:, 1], torch.randperm(N, generator=g)[:n].to(torch.int32)], 1)
    api.swap_blocks(in_pairs.to(cuda_dev), to_host=False, host_pool=host, pool=pool)
    oracle.swap_blocks(kc, vc, hk, hv, in_pairs, to_host=False)
    torch.cuda.synchronize()
    assert torch.equal(pool.k_pool.cpu(), kc) and torch.equal(pool.v_pool.cpu(), vc)
    assert pool.check_device_errors() == 0


def test_swap_blocks_checks_ids_and_host_memory(cuda_dev):
    pool = api.kv_pool_create(16, 16, 2, 64, torch.bfloat16, cuda_dev)
    _random_pool(pool, 13)
    host = api.host_pool_create(4, pool)
    before = host.k.clone()
    # a host id outside the host pool is recorded and skipped, nothing written
    api.swap_blocks(torch.tensor([[3, 4], [2, -1]], dtype=torch.int32, device=cuda_dev), to_host=True,
                    host_pool=host, pool=pool)
    torch.cuda.synchronize()
    assert pool.check_device_errors() == 5            # PK_ERR_BAD_INDEX
    assert torch.equal(host.k, before)
    # pageable host memory has no device mapping: refused before any launch
    pageable = api.HostPool.__new__(api.HostPool)
    pageable.k, pageable.v, pageable.num_blocks = torch.zeros_like(host.k), torch.zeros_like(host.v), 4
    assert not pageable.k.is_pinned()
    with pytest.raises(api.PagedKVError) as e:
        api.swap_blocks(torch.tensor([[0, 0]], dtype=torch.int32, device=cuda_dev), to_host=True,
                        host_pool=pageable, pool=pool)
    assert "mapped" in str(e.value)
