"""Pins for the float64 attention oracle (CPU only).

Each check ties the oracle to something other than itself:
  * torch's scaled_dot_product_attention (a library routine) on the same
    logical tokens held contiguously: paging must not change attention
    [PagedAttention & Continuous Batching (study notes), "Block tables"];
  * bit-identical results under different random permutations of the
    physical block ids (the table is the only thing that changes);
  * closed forms: one visible key returns its value; equal keys or a zero
    query average the visible values; a two-key case worked by hand;
  * chunked prefill equals the same tokens decoded one at a time
    [Batching and PagedAttention, "Continuous batching": chunks are split
    across steps, so the split must not change the answer];
  * GQA grouping with constant per-head values.
"""

import math

import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_chunked_b200.workloads import contiguous_to_paged, make_batch


def _sdpa_reference(q_rows, k_seq, v_seq, qlens, n_q_heads):
    """torch SDPA (float64) per sequence, causal with the chunk at the end of
    the context, GQA by repeating kv heads."""
    outs, t0 = [], 0
    for b, (k, v) in enumerate(zip(k_seq, v_seq)):
        qb = q_rows[t0:t0 + qlens[b]]
        t0 += qlens[b]
        c, Hkv, d = k.shape
        g = n_q_heads // Hkv
        kk = k.transpose(0, 1).repeat_interleave(g, dim=0)   # [Hq, c, d]
        vv = v.transpose(0, 1).repeat_interleave(g, dim=0)
        qq = qb.transpose(0, 1)                               # [Hq, q, d]
        pos_q = torch.arange(c - qlens[b], c)[:, None]
        pos_k = torch.arange(c)[None, :]
        mask = pos_k <= pos_q                                 # [q, c]
        o = F.scaled_dot_product_attention(qq[None], kk[None], vv[None], attn_mask=mask[None, None],
                                           scale=1.0 / math.sqrt(d))
        outs.append(o[0].transpose(0, 1))
    return torch.cat(outs, 0)


CASES = [
    # context lens, query lens, Hq, Hkv, d, block size
    ([5, 16, 17, 40], [1, 1, 1, 1], 8, 8, 64, 16),
    ([1, 2, 3, 33], [1, 2, 3, 7], 4, 2, 16, 4),
    ([19, 64, 7], [19, 8, 1], 7, 1, 8, 8),
    ([50, 31], [13, 31], 8, 2, 32, 1),
    ([100], [100], 16, 4, 8, 32),
]


@pytest.mark.parametrize("ctx,qlens,Hq,Hkv,d,bs", CASES)
def test_oracle_matches_sdpa_on_contiguous_tokens(ctx, qlens, Hq, Hkv, d, bs):
    g = torch.Generator().manual_seed(11)
    k_seq = [torch.randn((c, Hkv, d), generator=g, dtype=torch.float64) for c in ctx]
    v_seq = [torch.randn((c, Hkv, d), generator=g, dtype=torch.float64) for c in ctx]
    q = torch.randn((sum(qlens), Hq, d), generator=g, dtype=torch.float64)
    k_pool, v_pool, tables = contiguous_to_paged(k_seq, v_seq, bs, seed=5)
    qsl = torch.tensor([0] + list(torch.cumsum(torch.tensor(qlens), 0)), dtype=torch.int32)
    got = oracle.paged_attention(q, k_pool, v_pool, tables, torch.tensor(ctx), qsl, 1 / math.sqrt(d))
    ref = _sdpa_reference(q, k_seq, v_seq, qlens, Hq)
    assert torch.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_permuted_block_ids_give_identical_results():
    ctx, qlens = [37, 3, 64], [5, 1, 16]
    g = torch.Generator().manual_seed(3)
    k_seq = [torch.randn((c, 2, 16), generator=g, dtype=torch.float64) for c in ctx]
    v_seq = [torch.randn((c, 2, 16), generator=g, dtype=torch.float64) for c in ctx]
    q = torch.randn((sum(qlens), 4, 16), generator=g, dtype=torch.float64)
    qsl = torch.tensor([0, 5, 6, 22], dtype=torch.int32)
    outs = []
    for seed in range(6):
        k_pool, v_pool, tables = contiguous_to_paged(k_seq, v_seq, 8, seed=seed, num_blocks=20)
        outs.append(oracle.paged_attention(q, k_pool, v_pool, tables, torch.tensor(ctx), qsl, 0.25))
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_single_visible_key_returns_its_value():
    # c = 1: softmax over one score is exactly 1, so out = v_0 bit for bit
    b = make_batch([1, 1], None, block_size=16, n_q_heads=4, n_kv_heads=2, head_dim=8,
                   dtype=torch.float64, seed=2)
    out = oracle.paged_attention(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                 b["context_lens"], b["query_start_lens"], b["scale"])
    for s in range(2):
        blk = int(b["block_tables"][s, 0])
        for h in range(4):
            assert torch.equal(out[s, h], b["v_pool"][blk, h // 2, 0])


def test_equal_keys_and_zero_query_average_the_values():
    b = make_batch([23, 9], [4, 1], block_size=4, n_q_heads=2, n_kv_heads=1, head_dim=8,
                   dtype=torch.float64, seed=4)
    k_pool = torch.ones_like(b["k_pool"]) * 0.7          # every key identical
    out = oracle.paged_attention(b["q"], k_pool, b["v_pool"], b["block_tables"],
                                 b["context_lens"], b["query_start_lens"], b["scale"])
    zero_q = oracle.paged_attention(torch.zeros_like(b["q"]), b["k_pool"].nan_to_num(0.0),
                                    b["v_pool"], b["block_tables"], b["context_lens"],
                                    b["query_start_lens"], b["scale"])
    qsl = b["query_start_lens"].tolist()
    for s, c in enumerate([23, 9]):
        tbl = b["block_tables"][s]
        vals = torch.stack([b["v_pool"][tbl[j // 4], 0, j % 4] for j in range(c)])
        qlen = qsl[s + 1] - qsl[s]
        for i in range(qlen):
            visible = c - qlen + i + 1
            mean = vals[:visible].mean(0)
            for h in range(2):
                assert torch.allclose(out[qsl[s] + i, h], mean, rtol=0, atol=1e-13)
                assert torch.allclose(zero_q[qsl[s] + i, h], mean, rtol=0, atol=1e-13)


def test_two_keys_by_hand():
    # q = (1, 0); k0 = (1, 0), k1 = (0, 0); scale = ln 3  ->  scores ln 3 and 0,
    # softmax weights 3/4 and 1/4.  v0 = (4, 0), v1 = (0, 8)  ->  out = (3, 2).
    k_pool = torch.zeros((2, 1, 2, 2), dtype=torch.float64)
    v_pool = torch.zeros_like(k_pool)
    k_pool[1, 0, 0] = torch.tensor([1.0, 0.0])   # logical token 0 lives in physical block 1
    v_pool[1, 0, 0] = torch.tensor([4.0, 0.0])
    v_pool[1, 0, 1] = torch.tensor([0.0, 8.0])
    q = torch.tensor([[[1.0, 0.0]]], dtype=torch.float64)
    out = oracle.paged_attention(q, k_pool, v_pool, torch.tensor([[1]]), torch.tensor([2]),
                                 torch.tensor([0, 1]), math.log(3.0))
    assert torch.allclose(out[0, 0], torch.tensor([3.0, 2.0], dtype=torch.float64), atol=1e-14)
    # the same query placed first in a 2-token chunk sees only key 0
    q2 = torch.cat([q, q])
    out2 = oracle.paged_attention(q2, k_pool, v_pool, torch.tensor([[1]]), torch.tensor([2]),
                                  torch.tensor([0, 2]), math.log(3.0))
    assert torch.equal(out2[0, 0], torch.tensor([4.0, 0.0], dtype=torch.float64))
    assert torch.allclose(out2[1, 0], torch.tensor([3.0, 2.0], dtype=torch.float64), atol=1e-14)


def test_chunk_equals_successive_decode_steps():
    c, qlen, bs = 45, 12, 8
    b = make_batch([c], [qlen], block_size=bs, n_q_heads=6, n_kv_heads=3, head_dim=16,
                   dtype=torch.float64, seed=9)
    chunk = oracle.paged_attention(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                   b["context_lens"], b["query_start_lens"], b["scale"])
    for i in range(qlen):
        step = oracle.paged_attention(b["q"][i:i + 1], b["k_pool"], b["v_pool"], b["block_tables"],
                                      torch.tensor([c - qlen + i + 1]), torch.tensor([0, 1]),
                                      b["scale"])
        assert torch.equal(step[0], chunk[i])


def test_gqa_groups_are_contiguous():
    # kv head 0 holds value -3 everywhere, kv head 1 holds 7: q heads 0-3 read
    # head 0, q heads 4-7 read head 1 (h / (Hq / Hkv)).
    b = make_batch([10, 30], [2, 1], block_size=16, n_q_heads=8, n_kv_heads=2, head_dim=4,
                   dtype=torch.float64, seed=1, poison_unused=False)
    v_pool = torch.empty_like(b["v_pool"])
    v_pool[:, 0] = -3.0
    v_pool[:, 1] = 7.0
    out = oracle.paged_attention(b["q"], b["k_pool"], v_pool, b["block_tables"],
                                 b["context_lens"], b["query_start_lens"], b["scale"])
    assert torch.allclose(out[:, :4], torch.full_like(out[:, :4], -3.0), atol=1e-13)
    assert torch.allclose(out[:, 4:], torch.full_like(out[:, 4:], 7.0), atol=1e-13)


def test_sampled_rows_equal_full_batch():
    b = make_batch([40, 17, 64], [1, 17, 9], block_size=16, n_q_heads=4, n_kv_heads=1,
                   head_dim=32, dtype=torch.bfloat16, seed=13)
    full = oracle.paged_attention(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                  b["context_lens"], b["query_start_lens"], b["scale"])
    rows = [(0, 0), (5, 3), (26, 1), (17, 2)]
    part = oracle.paged_attention_rows(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                       b["context_lens"], b["query_start_lens"], b["scale"], rows)
    for i, (t, h) in enumerate(rows):
        assert torch.equal(part[i], full[t, h])


def test_rejects_bad_batches():
    b = make_batch([5], [1], block_size=4, n_q_heads=2, n_kv_heads=1, head_dim=4,
                   dtype=torch.float32, seed=0)
    args = (b["q"], b["k_pool"], b["v_pool"])
    with pytest.raises(ValueError):   # more queries than context
        oracle.paged_attention(torch.cat([b["q"]] * 6), *args[1:], b["block_tables"],
                               torch.tensor([5]), torch.tensor([0, 6]), 1.0)
    bad = b["block_tables"].clone()
    bad[0, 1] = b["num_blocks"]
    with pytest.raises(ValueError):   # block id outside the pool
        oracle.paged_attention(*args, bad, b["context_lens"], b["query_start_lens"], 1.0)
