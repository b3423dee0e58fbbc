"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no attention, no allocation policy).  Physical block ids
are a seeded random permutation of the pool, so a sequence's blocks are
scattered the way an allocator under churn leaves them [Batching and
PagedAttention, "PagedAttention": blocks live anywhere in GPU memory].

Workloads (sizes as the spec configurations name them):
  tiny_fp32      4 decode sequences, contexts {5, 16, 17, 40}, block 16, pool of
                 32 blocks, 8 q / 8 kv heads, head dim 64, float32, scale 1/8
  decode64_bf16  64 decode sequences, contexts uniform in [128, 4096], block 16,
                 32 q / 8 kv heads, head dim 128, pool 1.25x the blocks needed
  longdoc_bf16   8 decode sequences of 32,768 tokens, block 16, 16 q / 4 kv
                 heads, head dim 256, pool 1.25x
  chunk512_bf16  16 sequences at context 4096 whose last 512 tokens are this
                 step's prefill chunk (causal), 32 q / 8 kv heads, head dim 128
  chunk512_d256_bf16  the same chunks at head dim 256 with 16 q / 4 kv heads (the
                 long-document geometry)
  mixed_bf16     one continuous-batching step: 128 decode sequences with
                 contexts uniform in [128, 2048] and four 512-token prefill
                 chunks at contexts 1024, 2048, 3072 and 4096 (2,176 query
                 tokens), 32 q / 8 kv heads, head dim 128, block 16
"""

import math
import random

import torch

WORKLOADS = {
    "tiny_fp32": dict(context_lens=[5, 16, 17, 40], block_size=16, num_blocks=32, n_q_heads=8,
                      n_kv_heads=8, head_dim=64, dtype=torch.float32, seed=1001),
    "decode64_bf16": dict(num_seqs=64, ctx_range=(128, 4096), block_size=16, n_q_heads=32,
                          n_kv_heads=8, head_dim=128, dtype=torch.bfloat16, pool_factor=1.25,
                          seed=1002),
    "longdoc_bf16": dict(context_lens=[32768] * 8, block_size=16, n_q_heads=16, n_kv_heads=4,
                         head_dim=256, dtype=torch.bfloat16, pool_factor=1.25, seed=1003),
    # the last 512-token chunk of sixteen 4096-token prompts (chunked prefill)
    "chunk512_bf16": dict(context_lens=[4096] * 16, query_lens=[512] * 16, block_size=16,
                          n_q_heads=32, n_kv_heads=8, head_dim=128, dtype=torch.bfloat16,
                          pool_factor=1.25, seed=1006),
    "chunk512_d256_bf16": dict(context_lens=[4096] * 16, query_lens=[512] * 16, block_size=16,
                               n_q_heads=16, n_kv_heads=4, head_dim=256, dtype=torch.bfloat16,
                               pool_factor=1.25, seed=1009),
    # decodes first, then the chunks, the order the scheduler emits them
    "mixed_bf16": dict(num_seqs=128, ctx_range=(128, 2048), chunk_contexts=[1024, 2048, 3072, 4096],
                       chunk_len=512, block_size=16, n_q_heads=32, n_kv_heads=8, head_dim=128,
                       dtype=torch.bfloat16, pool_factor=1.25, seed=1008),
}


def page_toy_lengths(n=200, seed=7, mean=600, floor=50, max_len=4096):
    """Final request lengths of the capacity toy [Batching and PagedAttention,
    "Try it"]: seeded exponential draws (mean 600) shifted by 50 and capped at
    the longest allowed request."""
    rng = random.Random(seed)
    return [min(max_len, int(rng.expovariate(1.0 / mean)) + floor) for _ in range(n)]


def decode_context_lens(num_seqs, lo, hi, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (num_seqs,), generator=g).tolist()


def make_batch(context_lens, query_lens=None, *, block_size, n_q_heads, n_kv_heads, head_dim,
               dtype, seed, num_blocks=None, pool_factor=1.25, table_width=None,
               poison_unused=True, device="cpu", values="normal"):
    """A paged batch with scattered blocks.

    context_lens[b] tokens are stored for sequence b (the step's new tokens
    included); query_lens[b] (default 1: decode) of them are this step's
    queries.  Returns a dict with q [T, Hq, d], k_pool / v_pool [N, Hkv, bs, d],
    block_tables [B, W] int32 (-1 padded), context_lens [B] int32,
    query_start_lens [B + 1] int32 and scale = 1/sqrt(d).

    Unused pool blocks and the unwritten tail slots of each last block are
    filled with NaN when poison_unused is set, so that a kernel that reads
    past a sequence's context or through a wrong table entry cannot pass.
    """
    B = len(context_lens)
    if query_lens is None:
        query_lens = [1] * B
    g = torch.Generator().manual_seed(seed)
    nblk = [math.ceil(c / block_size) for c in context_lens]
    needed = sum(nblk)
    if num_blocks is None:
        num_blocks = max(needed, math.ceil(pool_factor * needed))
    if num_blocks < needed:
        raise ValueError("pool too small for the batch")
    width = table_width if table_width is not None else max(nblk + [1])
    perm = torch.randperm(num_blocks, generator=g)
    tables = torch.full((B, width), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        tables[b, :nblk[b]] = perm[pos:pos + nblk[b]].to(torch.int32)
        pos += nblk[b]

    shape = (num_blocks, n_kv_heads, block_size, head_dim)
    if values == "normal":
        k_pool = torch.randn(shape, generator=g, dtype=torch.float32)
        v_pool = torch.randn(shape, generator=g, dtype=torch.float32)
    else:
        raise ValueError(values)
    if poison_unused:
        used = torch.zeros((num_blocks, block_size), dtype=torch.bool)
        for b in range(B):
            for j in range(nblk[b]):
                n_in = min(block_size, context_lens[b] - j * block_size)
                used[tables[b, j], :n_in] = True
        mask = (~used)[:, None, :, None].expand(shape)
        k_pool[mask] = float("nan")
        v_pool[mask] = float("nan")
    T = sum(query_lens)
    q = torch.randn((T, n_q_heads, head_dim), generator=g, dtype=torch.float32)
    qsl = torch.zeros(B + 1, dtype=torch.int32)
    qsl[1:] = torch.cumsum(torch.tensor(query_lens, dtype=torch.int32), 0)
    return {
        "q": q.to(dtype).to(device),
        "k_pool": k_pool.to(dtype).to(device),
        "v_pool": v_pool.to(dtype).to(device),
        "block_tables": tables.to(device),
        "context_lens": torch.tensor(context_lens, dtype=torch.int32).to(device),
        "query_start_lens": qsl.to(device),
        "scale": 1.0 / math.sqrt(head_dim),
        "block_size": block_size,
        "num_blocks": num_blocks,
    }


def workload_batch(name, device="cpu", poison_unused=True):
    """The named decode workload (see the module docstring) as a batch."""
    w = dict(WORKLOADS[name])
    seed = w.pop("seed")
    if "num_seqs" in w:
        lo, hi = w.pop("ctx_range")
        ctx = decode_context_lens(w.pop("num_seqs"), lo, hi, seed)
    else:
        ctx = w.pop("context_lens")
    ql = w.pop("query_lens", None)
    if "chunk_contexts" in w:
        chunks, n = w.pop("chunk_contexts"), w.pop("chunk_len")
        ql = [1] * len(ctx) + [n] * len(chunks)
        ctx = list(ctx) + list(chunks)
    return make_batch(ctx, ql, seed=seed, device=device, poison_unused=poison_unused, **w)


def contiguous_to_paged(k_seq, v_seq, block_size, seed, num_blocks=None):
    """Scatter per-sequence contiguous K/V ([c_b, Hkv, d] each) into a pool
    with randomly permuted physical blocks.  Used to test that paging leaves
    attention unchanged.  Returns (k_pool, v_pool, block_tables)."""
    g = torch.Generator().manual_seed(seed)
    B = len(k_seq)
    Hkv, d = k_seq[0].shape[1], k_seq[0].shape[2]
    nblk = [math.ceil(k.shape[0] / block_size) for k in k_seq]
    needed = sum(nblk)
    num_blocks = num_blocks or needed + 3
    perm = torch.randperm(num_blocks, generator=g)
    k_pool = torch.full((num_blocks, Hkv, block_size, d), float("nan"), dtype=k_seq[0].dtype)
    v_pool = torch.full_like(k_pool, float("nan"))
    tables = torch.full((B, max(nblk)), -1, dtype=torch.int32)
    pos = 0
    for b in range(B):
        for j in range(nblk[b]):
            blk = int(perm[pos])
            pos += 1
            tables[b, j] = blk
            lo, hi = j * block_size, min((j + 1) * block_size, k_seq[b].shape[0])
            k_pool[blk, :, :hi - lo, :] = k_seq[b][lo:hi].transpose(0, 1)
            v_pool[blk, :, :hi - lo, :] = v_seq[b][lo:hi].transpose(0, 1)
    return k_pool, v_pool, tables


# ---------------------------------------------------------------- trace inputs
def _mix64(x):
    """SplitMix64 finaliser on int64 tensors (wrapping arithmetic): a
    counter-based generator, so a token's values depend only on its key."""
    x = x ^ ((x >> 30) & 0x3FFFFFFFF)
    x = x * -4658895280553007687          # 0xbf58476d1ce4e5b9 as a signed int64
    x = x ^ ((x >> 27) & 0x1FFFFFFFFF)
    x = x * -7723592293110705685          # 0x94d049bb133111eb as a signed int64
    x = x ^ ((x >> 31) & 0x1FFFFFFFF)
    return x


_TABLE_ROWS = 1 << 14
_tables = {}


def _value_table(seed, stream, n_heads, head_dim, dtype, device):
    """A seeded table of _TABLE_ROWS rows of N(0, 1) values [rows, n_heads,
    head_dim], drawn on the CPU (so every device holds the same bits) and kept."""
    device = torch.device(device)
    key = (seed, stream, n_heads, head_dim, dtype, device)
    t = _tables.get(key)
    if t is None:
        cpu_key = (seed, stream, n_heads, head_dim, dtype, torch.device("cpu"))
        t = _tables.get(cpu_key)
        if t is None:
            g = torch.Generator().manual_seed((seed * 1000003 + stream) * 7919 + n_heads * 1009 + head_dim)
            t = torch.randn((_TABLE_ROWS, n_heads, head_dim), generator=g).to(dtype)
            _tables[cpu_key] = t
        t = t.to(device)
        _tables[key] = t
    return t


def token_values(seed, stream, rids, positions, n_heads, head_dim, dtype, device="cpu"):
    """Deterministic pseudo-normal values for (request id, position) pairs:
    [len(positions), n_heads, head_dim].  stream separates q / k / v.

    A counter-based hash (SplitMix64 finaliser) of (seed, stream, request id,
    position) picks one row of a seeded N(0, 1) table, so a token's values
    depend only on its key, CPU and GPU produce the same bits, and one gather
    on the device makes a whole step's values.  Used so that a preempted
    request recomputes exactly the K/V it had."""
    rids = torch.as_tensor(rids, dtype=torch.int64)
    pos = torch.as_tensor(positions, dtype=torch.int64)
    key = ((seed * 1000003 + stream) * 1000003 + rids) * 1048576 + pos
    rows = _mix64(key) & (_TABLE_ROWS - 1)
    table = _value_table(seed, stream, n_heads, head_dim, dtype, device)
    if table.is_cuda:
        rows = rows.pin_memory()   # a copy from pageable memory would wait for the stream
    return table.index_select(0, rows.to(table.device, non_blocking=True))


def token_values_qkv(seed, rids, positions, n_q_heads, n_kv_heads, head_dim, dtype, device="cpu"):
    """token_values of streams 0, 1 and 2 (q, k, v) for the same keys, with one
    hash pass over a [3, T] key tensor and one host-to-device copy of the rows:
    the same values as three token_values calls."""
    rids = torch.as_tensor(rids, dtype=torch.int64)
    pos = torch.as_tensor(positions, dtype=torch.int64)
    streams = torch.arange(3, dtype=torch.int64)[:, None]
    key = ((seed * 1000003 + streams) * 1000003 + rids[None, :]) * 1048576 + pos[None, :]
    rows = _mix64(key) & (_TABLE_ROWS - 1)
    tables = [_value_table(seed, st, h, head_dim, dtype, device)
              for st, h in ((0, n_q_heads), (1, n_kv_heads), (2, n_kv_heads))]
    if tables[0].is_cuda:
        rows = rows.pin_memory()   # a copy from pageable memory would wait for the stream
    rows = rows.to(tables[0].device, non_blocking=True)
    return tuple(t.index_select(0, rows[i]) for i, t in enumerate(tables))


def trace_requests(n_steps=300, arrivals_per_step=4.0, prompt_median=512, prompt_sigma=1.0,
                   prompt_max=8192, out_min=10, out_max=500, seed=1004):
    """Continuous-batching trace: Poisson arrivals per step, lognormal prompt
    lengths (median prompt_median, clipped to [1, prompt_max]), output lengths
    uniform in [out_min, out_max].  Returns a list of (arrival_step, prompt_len,
    output_len) in arrival order.  Lengths are mixed on purpose: equal lengths
    hide what continuous batching is for ["Batching and PagedAttention",
    "Common mistakes"]."""
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for step in range(n_steps):
        for _ in range(int(rng.poisson(arrivals_per_step))):
            p = int(round(float(rng.lognormal(math.log(prompt_median), prompt_sigma))))
            p = min(max(p, 1), prompt_max)
            o = int(rng.integers(out_min, out_max + 1))
            out.append((step, p, o))
    return out


# value ids at or above this are shared system prompts, not requests
SYS_VID_BASE = 1 << 30


def prefix_trace_requests(n_steps=300, arrivals_per_step=4.0, sys_lens=(1024, 512, 2048, 256),
                          user_median=256, user_sigma=1.0, user_max=4096, out_min=10, out_max=500,
                          seed=1007):
    """A continuous-batching trace in which every request starts with one of a
    few shared system prompts ["Batching and PagedAttention", "Sharing
    blocks": requests that share a system prompt can share its blocks]:
    Poisson arrivals, a system prompt drawn uniformly from sys_lens, then a
    lognormal user part (median user_median, clipped to [1, user_max]) and an
    output length uniform in [out_min, out_max].  Returns (arrival_step,
    prompt_len, output_len, group, sys_len) tuples in arrival order; a
    request's tokens before sys_len are its group's, the rest its own."""
    import numpy as np
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for step in range(n_steps):
        for _ in range(int(rng.poisson(arrivals_per_step))):
            g = int(rng.integers(0, len(sys_lens)))
            u = int(round(float(rng.lognormal(math.log(user_median), user_sigma))))
            u = min(max(u, 1), user_max)
            o = int(rng.integers(out_min, out_max + 1))
            out.append((step, sys_lens[g] + u, o, g, sys_lens[g]))
    return out
