"""pk_paged_attention_append: the query rows' own K/V stored at their positions,
then attention, in one call.

Each case runs twice on copies of the same pool:
- once as pk_paged_kv_append, with the slots the block tables give, followed by
  pk_paged_attention;
- once as the fused call.

The two pools must match bit for bit. The two outputs must be bit-identical,
because the same attention kernels read the same values. The fused output must
also match the float64 oracle on the appended pool, within the bf16 tolerance.

The cases cover every path of the call:
- the block-streaming decode kernel, which stores decode rows just before it
  loads their blocks and, in a mixed step, the chunk rows before the chunk
  kernel starts;
- the position append kernel in front of the tile-streaming decode, mma.sync
  chunk and general kernels.
"""

import pytest
import torch

from paged_kv_cache_chunked_b200 import api
from paged_kv_cache_chunked_b200.workloads import make_batch

from helpers import assert_close, gpu_pool_from, oracle_attention

pytestmark = pytest.mark.gpu

CASES = [
    # contexts, query lengths, Hq, Hkv, d, block size, dtype, what
    ([1, 17, 300, 1029, 4000] * 4, None, 32, 8, 128, 16, torch.bfloat16, "decode, block-streaming"),
    ([5000, 20, 2100, 777], None, 16, 4, 256, 16, torch.bfloat16, "decode d 256, merge kernel"),
    ([3, 64, 65, 900], None, 8, 8, 64, 16, torch.bfloat16, "decode d 64"),
    ([400, 1300, 70, 2000, 33, 600], [1, 130, 1, 512, 1, 3], 32, 8, 128, 16, torch.bfloat16,
     "mixed decodes and chunks"),
    ([700, 2048], [256, 512], 32, 8, 128, 16, torch.bfloat16, "chunks only"),
    ([300, 45, 1111], None, 32, 2, 128, 16, torch.bfloat16, "decode, 16 q heads per kv head"),
    ([100, 260], [1, 40], 32, 8, 128, 8, torch.bfloat16, "mixed, block size 8"),
    ([50, 333, 9], [1, 7, 1], 8, 8, 64, 16, torch.float32, "fp32 pool"),
    ([100, 700, 33, 1], None, 32, 8, 128, 32, torch.bfloat16, "decode, block size 32"),
    ([50, 3000, 129], [1, 200, 64], 16, 4, 128, 64, torch.bfloat16, "mixed, block size 64"),
    ([1 + (i * 53) % 300 for i in range(600)], None, 8, 2, 64, 16, torch.bfloat16,
     "600 sequences, two launch windows"),
    ([max(64, 1 + (i * 53) % 300) for i in range(600)], [40 if i % 50 == 0 else 1 for i in range(600)],
     32, 8, 128, 16, torch.bfloat16, "600 sequences with chunks, two launch windows"),
]


def _same_bits(a, b):
    """Bit-for-bit equality (NaN in the poisoned slots included)."""
    it = torch.int16 if a.element_size() == 2 else torch.int32
    return torch.equal(a.view(it), b.view(it))


def _slots(batch):
    """Slot of every query row: position c_b - q_b + i of its sequence."""
    qsl = batch["query_start_lens"].tolist()
    ctx = batch["context_lens"].tolist()
    bs = batch["block_size"]
    tables = batch["block_tables"]
    out = []
    for b, c in enumerate(ctx):
        q = qsl[b + 1] - qsl[b]
        for i in range(q):
            pos = c - q + i
            out.append(int(tables[b, pos // bs]) * bs + pos % bs)
    return torch.tensor(out, dtype=torch.int64)


@pytest.mark.parametrize("ctx,ql,Hq,Hkv,d,bs,dtype,what", CASES, ids=[c[-1] for c in CASES])
def test_fused_append_equals_append_then_attention(cuda_dev, ctx, ql, Hq, Hkv, d, bs, dtype, what):
    b = make_batch(ctx, ql, block_size=bs, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, dtype=dtype, seed=61)
    T = b["q"].shape[0]
    g = torch.Generator().manual_seed(62)
    k_new = torch.randn((T, Hkv, d), generator=g).to(dtype)
    v_new = torch.randn((T, Hkv, d), generator=g).to(dtype)
    slots = _slots(b)
    dev = cuda_dev
    q = b["q"].to(dev)
    bt, dctx, dqsl = b["block_tables"].to(dev), b["context_lens"].to(dev), b["query_start_lens"].to(dev)
    dk, dv = k_new.to(dev), v_new.to(dev)

    pool_a = gpu_pool_from(b, Hkv, d, dtype, dev)
    api.paged_kv_append(dk, dv, slots.to(dev), pool=pool_a)
    out_a = api.paged_attention(q, pool_a.k_pool, pool_a.v_pool, bt, dctx, dqsl, b["scale"])

    pool_b = gpu_pool_from(b, Hkv, d, dtype, dev)
    out_b = api.paged_attention_append(q, dk, dv, pool_b.k_pool, pool_b.v_pool, bt, dctx, dqsl, b["scale"])
    torch.cuda.synchronize(dev)

    assert _same_bits(pool_a.k_pool, pool_b.k_pool), what
    assert _same_bits(pool_a.v_pool, pool_b.v_pool), what
    assert _same_bits(out_a, out_b), what
    appended = dict(b)
    appended["k_pool"] = pool_b.k_pool.cpu()
    appended["v_pool"] = pool_b.v_pool.cpu()
    assert_close(out_b, oracle_attention(appended), dtype, what + " vs oracle")
    assert pool_a.check_device_errors() == 0 and pool_b.check_device_errors() == 0


def test_fused_append_back_to_back(cuda_dev):
    # Steps of one growing decode batch issued without a synchronisation between
    # them: each step appends one token per sequence and attends over it. The
    # next step's kernels start while the previous step drains, so this checks
    # that a row is stored before its block is loaded and never overwritten
    # late. The final pool and every step's output must equal the separate calls.
    Hq, Hkv, d, bs, steps = 32, 8, 128, 16, 5
    base = [40 + (i * 113) % 900 for i in range(48)]
    full = make_batch([c + steps for c in base], None, block_size=bs, n_q_heads=Hq, n_kv_heads=Hkv,
                      head_dim=d, dtype=torch.bfloat16, seed=63, poison_unused=False)
    g = torch.Generator().manual_seed(64)
    dev = cuda_dev
    pool_a = gpu_pool_from(full, Hkv, d, torch.bfloat16, dev)
    pool_b = gpu_pool_from(full, Hkv, d, torch.bfloat16, dev)
    bt = full["block_tables"].to(dev)
    qsl = torch.arange(len(base) + 1, dtype=torch.int32, device=dev)
    outs_a, outs_b, inputs = [], [], []
    for s in range(steps):
        ctx = torch.tensor([c + s + 1 for c in base], dtype=torch.int32)
        q = torch.randn((len(base), Hq, d), generator=g).to(torch.bfloat16)
        k = torch.randn((len(base), Hkv, d), generator=g).to(torch.bfloat16)
        v = torch.randn((len(base), Hkv, d), generator=g).to(torch.bfloat16)
        step_batch = dict(full, context_lens=ctx, query_start_lens=qsl.cpu())
        inputs.append((q.to(dev), k.to(dev), v.to(dev), ctx.to(dev), _slots(step_batch).to(dev)))
    torch.cuda.synchronize(dev)
    for q, k, v, ctx, slots in inputs:
        api.paged_kv_append(k, v, slots, pool=pool_a)
        outs_a.append(api.paged_attention(q, pool_a.k_pool, pool_a.v_pool, bt, ctx, qsl, full["scale"]))
    for q, k, v, ctx, slots in inputs:
        outs_b.append(api.paged_attention_append(q, k, v, pool_b.k_pool, pool_b.v_pool, bt, ctx, qsl,
                                                 full["scale"]))
    torch.cuda.synchronize(dev)
    assert _same_bits(pool_a.k_pool, pool_b.k_pool) and _same_bits(pool_a.v_pool, pool_b.v_pool)
    for s, (oa, ob) in enumerate(zip(outs_a, outs_b)):
        assert _same_bits(oa, ob), f"step {s}"
    assert pool_b.check_device_errors() == 0
