"""Capacity arithmetic the pages print (test infrastructure only).

* token-slot toy [Batching and PagedAttention, "Try it", the capacity script
  and its printed output]: a cache of a fixed number of token slots admits
  requests in arrival order until the next one does not fit; reserving the
  maximum length per request is compared with 16-token paging.  Paging here
  runs through the oracle block manager, so the printed figures pin it.
* KV bytes [7.8 PagedAttention & continuous batching (LLM deep dive),
  "01 Concept"]: bytes per token = layers x 2 (K and V) x kv heads x head
  dim x element bytes; a block holds block_size tokens; a session costs its
  tokens' KV plus any fixed per-sequence state; a pool holds the floor of
  pool / per-session sessions.
"""

from .allocator import OracleBlockManager, OracleOOM


def admit_reserve_max(lengths, capacity_slots, max_len):
    """Contiguous reservation of max_len slots per request, in order, until the
    next request does not fit.  Returns (admitted, used_slots, real_tokens)."""
    used = n = 0
    for _ in lengths:
        if used + max_len > capacity_slots:
            break
        used += max_len
        n += 1
    return n, used, sum(lengths[:n])


def admit_paged(lengths, capacity_slots, block_size):
    """Paged admission through the block manager: every request asks for its
    whole length; admission stops at the first allocation failure.
    Returns (admitted, used_slots, real_tokens)."""
    bm = OracleBlockManager(capacity_slots // block_size, block_size)
    n = 0
    for length in lengths:
        seq = bm.add_seq()
        try:
            bm.append_slots(seq, length)
        except OracleOOM:
            bm.free(seq)
            break
        n += 1
    return n, bm.num_used() * block_size, sum(lengths[:n])


def mean_tail_waste(lengths, block_size):
    """Average unwritten slots per request when every request is stored in its
    own blocks (pool large enough for all of them)."""
    total_blocks = sum(-(-length // block_size) for length in lengths)
    bm = OracleBlockManager(total_blocks, block_size)
    for length in lengths:
        bm.append_slots(bm.add_seq(), length)
    return bm.tail_waste() / len(lengths)


def kv_bytes_per_token(n_layers, n_kv_heads, head_dim, elt_bytes):
    """K and V bytes one token occupies across n_layers attention layers."""
    return n_layers * 2 * n_kv_heads * head_dim * elt_bytes


def block_bytes(block_size, bytes_per_token):
    return block_size * bytes_per_token


def sessions_in_pool(pool_bytes, tokens, bytes_per_token, fixed_state_bytes=0):
    """How many sessions of `tokens` tokens a pool holds when each is paged
    (its KV plus a fixed per-sequence state)."""
    return pool_bytes // (tokens * bytes_per_token + fixed_state_bytes)
