"""GPU parity of paged attention against the float64 oracle.

Tolerance: |gpu - oracle| <= 2e-2 + 2e-2 |oracle| for bf16 inputs with fp32
accumulation, 1e-4 + 1e-4 |oracle| for fp32 inputs, element by element.
Pools are seeded N(0, 1); every slot no sequence owns (unused blocks, the
tail of each last block) holds NaN, so reading past a context or through a
wrong table entry fails the test.
"""

import math
import os

import pytest
import torch

import oracle
from paged_kv_cache_chunked_b200 import api
from paged_kv_cache_chunked_b200.workloads import make_batch, workload_batch, contiguous_to_paged

from helpers import (assert_close, gpu_pool_from, oracle_attention, run_gpu_attention,
                     sample_rows)

pytestmark = pytest.mark.gpu


def _check(batch, Hq, Hkv, d, dtype, dev, what):
    pool = gpu_pool_from(batch, Hkv, d, dtype, dev)
    got = run_gpu_attention(batch, pool, dev)
    ref = oracle_attention(batch)
    err = assert_close(got, ref, dtype, what)
    assert pool.check_device_errors() == 0
    return got, err


def test_tiny_fp32_decode(cuda_dev):
    # 4 decode sequences, contexts {5, 16, 17, 40}, block 16, 32-block pool,
    # 8 q / 8 kv heads, head dim 64, float32, scale 1/8
    b = workload_batch("tiny_fp32")
    _check(b, 8, 8, 64, torch.float32, cuda_dev, "tiny fp32")


def test_tiny_fp32_as_causal_chunks(cuda_dev):
    # the same contexts processed as 8-token causal chunks (the last 8 tokens
    # of each context are queries; context 5 takes all 5)
    ctx = [5, 16, 17, 40]
    b = make_batch(ctx, [min(8, c) for c in ctx], block_size=16, num_blocks=32, n_q_heads=8,
                   n_kv_heads=8, head_dim=64, dtype=torch.float32, seed=1001)
    _check(b, 8, 8, 64, torch.float32, cuda_dev, "tiny fp32 chunks")


DECODE_CASES = [
    # contexts, Hq, Hkv, d, block size
    ([1, 2, 15, 16, 17, 31, 33, 100, 257, 600], 32, 8, 128, 16),
    ([5, 77, 300, 1029], 16, 4, 256, 16),
    ([3, 64, 65, 900], 8, 8, 64, 16),
    ([9, 120, 513], 32, 8, 128, 8),
    ([40, 700, 1], 32, 8, 128, 32),
    ([50, 333], 28, 4, 128, 16),      # group of 7
    ([21, 400], 16, 1, 128, 16),      # group of 16
    ([30, 250], 32, 1, 128, 16),      # group of 32: two row tiles per token
    ([64, 1000], 8, 8, 128, 16),      # group of 1
    # decode batches on the block-streaming kernel: every stage geometry
    ([30, 700, 2000], 8, 1, 128, 16),   # one kv head: eight phases per head, 8 blocks a stage
    ([100, 1500, 7], 2, 1, 64, 16),     # one kv head, d 64: 16 blocks a stage
    ([300, 50, 1200], 8, 2, 128, 16),   # two kv heads: four phases per head
    ([100, 800], 24, 6, 128, 16),       # six kv heads: three head groups of two
    ([500, 77], 32, 16, 64, 16),        # sixteen kv heads: two head groups of eight
    ([200, 3000], 4, 2, 256, 64),       # block 64, d 256: one head a stage
    ([90, 1000], 8, 8, 128, 256),       # block 256: too big for a stage, tile kernel instead
]


@pytest.mark.parametrize("ctx,Hq,Hkv,d,bs", DECODE_CASES)
def test_bf16_decode(cuda_dev, ctx, Hq, Hkv, d, bs):
    b = make_batch(ctx, None, block_size=bs, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                   dtype=torch.bfloat16, seed=sum(ctx) + d)
    _check(b, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"decode {ctx}")


CHUNK_CASES = [
    # contexts, query lens, Hq, Hkv, d, block size
    ([300, 200, 100, 50], [1, 64, 100, 3], 32, 8, 128, 16),
    ([1000, 513], [512, 17], 32, 8, 128, 16),
    ([129, 64], [129, 64], 16, 4, 256, 16),
    ([90, 45], [33, 45], 8, 8, 64, 8),
    ([600], [250], 28, 4, 128, 32),
    ([70, 18], [70, 5], 32, 1, 128, 16),
    # d 128, blocks of 16k: the tcgen05 chunk kernel, 256-row items of two 128-row tiles
    ([512], [512], 8, 8, 128, 16),               # g 1, a whole prompt as one chunk (no prior context)
    ([700, 300], [300, 129], 16, 8, 128, 16),    # g 2, ragged last row tile
    ([1100, 96], [600, 96], 64, 8, 128, 32),     # g 8, block 32
    ([2000, 40], [257, 40], 32, 2, 128, 64),     # g 16, block 64
    ([333, 20], [200, 1], 64, 1, 128, 16),       # g 64: one token fills 64 rows; a decode in the batch
    # d 64, blocks of 16k: the same tcgen05 kernel with one 64-column panel
    ([600, 77, 900], [300, 77, 1], 16, 4, 64, 16),   # g 4, a decode row on the block-streaming kernel
    ([1000], [512], 8, 8, 64, 32),                   # g 1, block 32
    ([333, 40], [200, 40], 64, 1, 64, 16),           # g 64
    # d 256: the tcgen05 kernel with one 128-row tile and two S buffers
    ([1500, 300, 900], [700, 300, 1], 16, 4, 256, 16),   # g 4, 64-key stages, a decode row
    ([1000], [257], 8, 8, 256, 32),                      # g 1, block 32
    ([400, 50], [200, 50], 64, 1, 256, 16),              # g 64
]


@pytest.mark.parametrize("ctx,ql,Hq,Hkv,d,bs", CHUNK_CASES)
def test_bf16_chunked_prefill_mixed_with_decode(cuda_dev, ctx, ql, Hq, Hkv, d, bs):
    b = make_batch(ctx, ql, block_size=bs, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                   dtype=torch.bfloat16, seed=7 + sum(ql))
    _check(b, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"chunks {ctx}/{ql}")


def test_decode_batch_over_several_launch_windows(cuda_dev):
    # 600 sequences: the kernels take 512 sequences a launch, so two windows
    ctx = [1 + (i * 37) % 90 for i in range(600)]
    b = make_batch(ctx, None, block_size=16, n_q_heads=8, n_kv_heads=2, head_dim=64,
                   dtype=torch.bfloat16, seed=77)
    _check(b, 8, 2, 64, torch.bfloat16, cuda_dev, "600 sequences")


def test_chunks_at_successive_offsets(cuda_dev):
    # a 900-token prompt as one chunk, and 300-token chunks at offsets 0, 300 and
    # 600 (each sees the earlier tokens as context): every row matches the oracle
    ctx_total, d, Hq, Hkv = 900, 128, 32, 8
    for start, qn in ((0, 900), (0, 300), (300, 300), (600, 300)):
        c = start + qn
        b = make_batch([c], [qn], block_size=16, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                       dtype=torch.bfloat16, seed=123)
        _check(b, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"chunk at {start}")


@pytest.mark.parametrize("ql", [[1, 40, 1, 33], [1, 1, 1, 1]], ids=["mixed", "decode_only"])
def test_permuted_block_ids_bit_identical(cuda_dev, ql):
    # paging must not change attention: same logical K/V under five different
    # physical permutations gives bit-identical GPU output, equal to the oracle
    # (mixed: chunk and tile-decode kernels; decode_only: block-streaming decode
    # kernel with its split-K merge)
    ctx, Hkv, Hq, d = [700, 90, 1500, 33], 8, 32, 128
    g = torch.Generator().manual_seed(21)
    k_seq = [torch.randn((c, Hkv, d), generator=g).to(torch.bfloat16) for c in ctx]
    v_seq = [torch.randn((c, Hkv, d), generator=g).to(torch.bfloat16) for c in ctx]
    q = torch.randn((sum(ql), Hq, d), generator=g).to(torch.bfloat16)
    qsl = torch.tensor([0] + torch.cumsum(torch.tensor(ql), 0).tolist(), dtype=torch.int32)
    outs = []
    for seed in range(5):
        kp, vp, tables = contiguous_to_paged(k_seq, v_seq, 16, seed=seed, num_blocks=200)
        batch = {"q": q, "k_pool": kp, "v_pool": vp, "block_tables": tables,
                 "context_lens": torch.tensor(ctx, dtype=torch.int32), "query_start_lens": qsl,
                 "scale": 1 / math.sqrt(d), "block_size": 16}
        got, _ = _check(batch, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"perm {seed}")
        outs.append(got.cpu())
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_split_k_merge_bit_identical_under_permutations(cuda_dev):
    # 48 decode rows of 8 kv heads on the block-streaming kernel: pairs cut
    # into partitions at chunk boundaries are combined by the merge kernel in
    # partition order, whatever CTA finished first, so the output is
    # bit-identical under any placement of the blocks, and equal to the oracle
    g = torch.Generator().manual_seed(31)
    ctx = torch.randint(200, 2500, (48,), generator=g).tolist()
    Hkv, Hq, d = 8, 32, 128
    k_seq = [torch.randn((c, Hkv, d), generator=g).to(torch.bfloat16) for c in ctx]
    v_seq = [torch.randn((c, Hkv, d), generator=g).to(torch.bfloat16) for c in ctx]
    q = torch.randn((len(ctx), Hq, d), generator=g).to(torch.bfloat16)
    qsl = torch.arange(len(ctx) + 1, dtype=torch.int32)
    outs = []
    for seed in range(3):
        kp, vp, tables = contiguous_to_paged(k_seq, v_seq, 16, seed=seed)
        batch = {"q": q, "k_pool": kp, "v_pool": vp, "block_tables": tables,
                 "context_lens": torch.tensor(ctx, dtype=torch.int32), "query_start_lens": qsl,
                 "scale": 1 / math.sqrt(d), "block_size": 16}
        got, _ = _check(batch, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"perm {seed}")
        outs.append(got.cpu())
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_back_to_back_calls_share_one_workspace(cuda_dev):
    # Calls on one pool and stream reuse one workspace: its split-K partial rows
    # and the merge kernel's list of split pairs.  A call's kernels start while
    # the previous call's merge kernel may still run, so four calls with
    # different split lists are issued without a synchronisation between them;
    # each must still match the oracle on its own sequences.
    full = make_batch([100 + (i * 389) % 3900 for i in range(96)], None, block_size=16,
                      n_q_heads=32, n_kv_heads=8, head_dim=128, dtype=torch.bfloat16, seed=34)
    pool = gpu_pool_from(full, 8, 128, torch.bfloat16, cuda_dev)
    subsets = [list(range(96)), list(range(0, 96, 3)), [5, 17, 60], list(range(40, 90))]
    outs, subs = [], []
    for idx in subsets:
        sub = dict(full)
        sub["q"] = full["q"][idx]
        sub["block_tables"] = full["block_tables"][idx]
        sub["context_lens"] = full["context_lens"][idx]
        sub["query_start_lens"] = torch.arange(len(idx) + 1, dtype=torch.int32)
        subs.append(sub)
    dev_in = [(s_["q"].to(cuda_dev), s_["block_tables"].to(cuda_dev), s_["context_lens"].to(cuda_dev),
               s_["query_start_lens"].to(cuda_dev)) for s_ in subs]
    torch.cuda.synchronize(cuda_dev)
    for _ in range(2):
        outs = [api.paged_attention(q, pool.k_pool, pool.v_pool, bt, ctx, qsl, full["scale"])
                for q, bt, ctx, qsl in dev_in]
    torch.cuda.synchronize(cuda_dev)
    for o, s_, idx in zip(outs, subs, subsets):
        assert_close(o, oracle_attention(s_), torch.bfloat16, f"{len(idx)} sequences, back to back")
    assert pool.check_device_errors() == 0


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (16, 4, 256)])
def test_chunk_order_past_the_rank_cap(cuda_dev, Hq, Hkv, d):
    # 300 sequences of 3-token chunks: more chunk sequences than the tcgen05
    # kernels rank by work (256), so their items are taken in window order;
    # every row against the oracle
    ctx = [20 + (i * 37) % 400 for i in range(300)]
    b = make_batch(ctx, [3] * len(ctx), block_size=16, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                   dtype=torch.bfloat16, seed=35)
    _check(b, Hq, Hkv, d, torch.bfloat16, cuda_dev, f"300 chunk sequences, d {d}")


def test_long_context_split_k(cuda_dev):
    # two 8k-token sequences with head dim 256: many split-K partitions
    b = make_batch([8192, 6000], None, block_size=16, n_q_heads=16, n_kv_heads=4, head_dim=256,
                   dtype=torch.bfloat16, seed=33)
    _check(b, 16, 4, 256, torch.bfloat16, cuda_dev, "long split-K")


@pytest.mark.parametrize("name", ["decode64_bf16", "longdoc_bf16"])
def test_full_size_decode_workloads_every_row(cuda_dev, name):
    # the bench's decode workloads at full size, in the launch configuration
    # the bench times: every output row against the oracle
    b = workload_batch(name, poison_unused=False)
    Hkv, d = b["k_pool"].shape[1], b["q"].shape[2]
    pool = gpu_pool_from(b, Hkv, d, torch.bfloat16, cuda_dev)
    got = run_gpu_attention(b, pool, cuda_dev)
    assert_close(got, oracle_attention(b), torch.bfloat16, name)
    assert pool.check_device_errors() == 0


@pytest.mark.parametrize("workload,item_rows", [("chunk512_bf16", 256), ("chunk512_d256_bf16", 128)])
def test_full_size_chunk512_sampled_rows(cuda_dev, workload, item_rows):
    # sixteen 512-token chunks at context 4,096 (the bench's prefill workloads,
    # head dim 128 and 256) at full size: the first and last row of every work
    # item of the tcgen05 kernel (256 rows at head dim 128, 128 at 256; rows are
    # (token, group head) pairs, token-major, per (sequence, kv head)) plus
    # 2,000 random rows, against the oracle
    b = workload_batch(workload, poison_unused=False)
    T, Hq, d = b["q"].shape
    Hkv = b["k_pool"].shape[1]
    g = Hq // Hkv
    pool = gpu_pool_from(b, Hkv, d, torch.bfloat16, cuda_dev)
    assert pool.paths() & api.PK_PATH_CHUNK_TCGEN05
    got = run_gpu_attention(b, pool, cuda_dev).cpu()
    rows = sample_rows(T, Hq, 2000, seed=6)
    qsl = b["query_start_lens"].tolist()
    for s in range(len(qsl) - 1):
        qn = qsl[s + 1] - qsl[s]
        for kvh in range(Hkv):
            for r0 in range(0, qn * g, item_rows):
                for r in (r0, min(r0 + item_rows - 1, qn * g - 1)):
                    rows.append([qsl[s] + r // g, kvh * g + r % g])
    ref = oracle.paged_attention_rows(b["q"], b["k_pool"], b["v_pool"], b["block_tables"],
                                      b["context_lens"], b["query_start_lens"], b["scale"], rows)
    got_rows = torch.stack([got[t, h] for t, h in rows])
    assert_close(got_rows, ref, torch.bfloat16, workload)
    assert torch.isfinite(got).all()
    assert pool.check_device_errors() == 0


@pytest.mark.parametrize("Hkv,d,bs,want", [
    (8, 128, 16, ("TENSOR_CORE", "DECODE_BLOCKS", "CHUNK_TCGEN05")),
    (4, 256, 16, ("TENSOR_CORE", "DECODE_BLOCKS", "CHUNK_TCGEN05")),
    (4, 256, 8, ("TENSOR_CORE", "DECODE_BLOCKS")),
    (8, 64, 16, ("TENSOR_CORE", "DECODE_BLOCKS", "CHUNK_TCGEN05")),
    (8, 128, 8, ("TENSOR_CORE", "DECODE_BLOCKS")),
])
def test_pool_paths(cuda_dev, Hkv, d, bs, want):
    # the kernels a pool selects are reported, so that losing the tcgen05 chunk
    # kernel (a register count other than the one its warp roles assume) is
    # seen rather than silently running every chunk on mma.sync
    pool = api.kv_pool_create(64, bs, Hkv, d, torch.bfloat16, cuda_dev)
    bits = {n: getattr(api, "PK_PATH_" + n) for n in ("TENSOR_CORE", "DECODE_BLOCKS", "CHUNK_TCGEN05")}
    assert {n for n, v in bits.items() if pool.paths() & v} == set(want)
    fp32 = api.kv_pool_create(64, 16, 8, 64, torch.float32, cuda_dev)
    assert fp32.paths() == 0


def test_single_token_context_returns_its_value(cuda_dev):
    b = make_batch([1, 1, 1], None, block_size=16, n_q_heads=8, n_kv_heads=2, head_dim=128,
                   dtype=torch.bfloat16, seed=4)
    pool = gpu_pool_from(b, 2, 128, torch.bfloat16, cuda_dev)
    got = run_gpu_attention(b, pool, cuda_dev).cpu()
    for s in range(3):
        blk = int(b["block_tables"][s, 0])
        for h in range(8):
            assert torch.equal(got[s, h], b["v_pool"][blk, h // 4, 0])


@pytest.mark.parametrize("ctx,ql,bs,d", [([37, 5], [4, 5], 4, 40), ([19], [19], 1, 16)])
def test_general_kernel_geometries(cuda_dev, ctx, ql, bs, d):
    # block sizes and head dims outside the tensor-core tiling run the general kernel
    b = make_batch(ctx, ql, block_size=bs, n_q_heads=4, n_kv_heads=2, head_dim=d,
                   dtype=torch.bfloat16, seed=3)
    _check(b, 4, 2, d, torch.bfloat16, cuda_dev, "general kernel")


def test_general_kernel_forced_on_bf16(cuda_dev):
    os.environ["PK_FORCE_GENERIC"] = "1"
    try:
        b = make_batch([300, 64], [1, 20], block_size=16, n_q_heads=32, n_kv_heads=8,
                       head_dim=128, dtype=torch.bfloat16, seed=8)
        _check(b, 32, 8, 128, torch.bfloat16, cuda_dev, "forced general")
    finally:
        del os.environ["PK_FORCE_GENERIC"]


def test_bad_block_id_is_recorded_not_dereferenced(cuda_dev):
    b = make_batch([40], None, block_size=16, n_q_heads=8, n_kv_heads=8, head_dim=128,
                   dtype=torch.bfloat16, seed=2, poison_unused=False)
    b["block_tables"][0, 1] = 10 ** 6
    pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
    run_gpu_attention(b, pool, cuda_dev)
    assert pool.check_device_errors() == 5


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (16, 4, 256)])
def test_split_k_partition_count_leaves_the_result_to_rounding(cuda_dev, Hq, Hkv, d):
    # One long decode sequence, alone, is cut into about a hundred split-K
    # partitions (one equal chunk of the stages per SM). Among 300 other
    # sequences, the same sequence, with the same pool, table and query, spans
    # only a few. The merge combines the partitions in fp32, but each partition
    # rounds its P to bf16 for the tensor core against its own reference max,
    # so the two outputs agree to P's rounding (2^-9 per weight) and the
    # output's own bf16 rounding, not to fp32: each (row, head) within 2^-6 of
    # its largest output magnitude (six seeds at d 128 and 256 reached at most
    # half of that). A merge that dropped or misweighted one of a hundred
    # partitions moves outputs by about a fifth of that magnitude.
    ctx = [8000] + [200 + (i * 97) % 1800 for i in range(300)]
    b = make_batch(ctx, None, block_size=16, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                   dtype=torch.bfloat16, seed=71, poison_unused=False)
    pool = gpu_pool_from(b, Hkv, d, torch.bfloat16, cuda_dev)
    many = run_gpu_attention(b, pool, cuda_dev)[0].float()
    alone = dict(b, q=b["q"][:1], block_tables=b["block_tables"][:1], context_lens=b["context_lens"][:1],
                 query_start_lens=b["query_start_lens"][:2])
    one = run_gpu_attention(alone, pool, cuda_dev)[0].float()
    bound = torch.maximum(many.abs(), one.abs()).amax(dim=-1, keepdim=True) * 2.0 ** -6
    assert ((many - one).abs() <= bound).all(), float(((many - one).abs() / bound).max())
    ref = oracle.paged_attention(alone["q"], b["k_pool"], b["v_pool"], alone["block_tables"],
                                 alone["context_lens"], alone["query_start_lens"], b["scale"])[0]
    assert_close(one, ref, torch.bfloat16, "alone")
    assert pool.check_device_errors() == 0
