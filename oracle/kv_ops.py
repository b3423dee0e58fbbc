"""Oracle for the two copy operations of the paged KV cache (test
infrastructure only).

kv_append
    "Append KV into mapped blocks" [PagedAttention & Continuous Batching
    (study notes), "Flow", step 4]: each new token's K and V rows are stored
    at the slot its block table maps it to.  Slot id reading: slot = physical
    block * block_size + offset inside the block; a negative slot means the
    token is not stored.
block_copy
    "A later write into a shared block allocates a fresh block, copies, then
    writes" [same page, "Copy-on-write"].  The copy moves the whole physical
    block (all heads, all slots, K and V).  All pairs of one call read the
    state from before the call.

Both work element by element on CPU torch tensors, in place.
"""

import torch


def kv_append(k_pool, v_pool, k, v, slot_mapping):
    """k_pool, v_pool: [num_blocks, n_kv_heads, block_size, head_dim];
    k, v: [num_tokens, n_kv_heads, head_dim]; slot_mapping: [num_tokens]."""
    num_blocks, n_kv_heads, block_size, head_dim = k_pool.shape
    slots = [int(s) for s in slot_mapping.tolist()]
    for t, s in enumerate(slots):
        if s < 0:
            continue
        block, offset = divmod(s, block_size)
        if block >= num_blocks:
            raise IndexError("slot outside the pool")
        for h in range(n_kv_heads):
            k_pool[block, h, offset, :] = k[t, h, :]
            v_pool[block, h, offset, :] = v[t, h, :]


def block_copy(k_pool, v_pool, src_dst_pairs):
    """src_dst_pairs: [n, 2] of (source block, destination block)."""
    pairs = [(int(a), int(b)) for a, b in torch.as_tensor(src_dst_pairs).reshape(-1, 2).tolist()]
    k_before = k_pool.clone()
    v_before = v_pool.clone()
    for src, dst in pairs:
        k_pool[dst] = k_before[src]
        v_pool[dst] = v_before[src]
