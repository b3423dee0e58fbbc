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
swap_blocks
    Whole blocks moved between the device pool and a host pool, the swap a
    preemption may use instead of recomputation.

All work on CPU torch tensors, in place.
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


def swap_blocks(k_pool, v_pool, host_k, host_v, pairs, to_host):
    """Whole-block moves between the device pool and a host pool of the same
    block geometry [Batching and PagedAttention, "When blocks run out": a
    preempted request's blocks are swapped out to CPU memory and later back].
    to_host: pairs are (device block, host block) and host[h] = pool[d];
    otherwise pairs are (host block, device block) and pool[d] = host[h].
    K and V alike."""
    pairs = [(int(a), int(b)) for a, b in torch.as_tensor(pairs).reshape(-1, 2).tolist()]
    for a, b in pairs:
        if to_host:
            host_k[b] = k_pool[a]
            host_v[b] = v_pool[a]
        else:
            k_pool[b] = host_k[a]
            v_pool[b] = host_v[a]
