"""Pins for the oracle append and block copy (CPU only): slot ids decompose
as physical block * block_size + offset, negative slots are skipped, a copy
moves whole blocks and reads the state from before the call."""

import torch

import oracle


def test_append_places_rows_by_slot():
    bs, Hkv, d = 4, 2, 3
    k_pool = torch.zeros((5, Hkv, bs, d))
    v_pool = torch.zeros_like(k_pool)
    k = torch.arange(3 * Hkv * d, dtype=torch.float32).reshape(3, Hkv, d) + 1
    v = -k
    slots = torch.tensor([13, -1, 2])       # block 3 offset 1; skipped; block 0 offset 2
    oracle.kv_append(k_pool, v_pool, k, v, slots)
    assert torch.equal(k_pool[3, :, 1], k[0]) and torch.equal(v_pool[3, :, 1], v[0])
    assert torch.equal(k_pool[0, :, 2], k[2]) and torch.equal(v_pool[0, :, 2], v[2])
    assert int((k_pool != 0).sum()) == 2 * Hkv * d      # nothing else written


def test_block_copy_moves_whole_blocks_from_the_old_state():
    k_pool = torch.arange(6 * 2 * 4 * 2, dtype=torch.float32).reshape(6, 2, 4, 2)
    v_pool = -k_pool
    k0, v0 = k_pool.clone(), v_pool.clone()
    oracle.block_copy(k_pool, v_pool, torch.tensor([[1, 4], [4, 5]]))
    assert torch.equal(k_pool[4], k0[1]) and torch.equal(v_pool[4], v0[1])
    assert torch.equal(k_pool[5], k0[4])      # reads the pre-call block 4
    for b in (0, 1, 2, 3):
        assert torch.equal(k_pool[b], k0[b])
