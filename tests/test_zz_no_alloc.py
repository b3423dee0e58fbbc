"""pk_paged_attention_noalloc: paged attention for callers that cannot
allocate device memory (a C host program with no caching allocator, a serving
loop that has reserved all free HBM for the KV pool).  It takes its scratch
from a fixed array inside the library instead of a caller workspace.

Checked through the C ABI against pk_paged_attention, on two calls in a row
(the second one finds the first one's leftovers in the shared array), within
the bf16 tolerance the other attention tests use, and against the float64
oracle; on pools of different kv-head counts one after the other (the shared
array's counters must sit where every pool looks for them); with the split-K
counters deliberately left non-zero (what a call that gave up on a bounded
wait could leave); and with no sequences at all.  This file is collected last
so that a failure here comes after every other test has run.
"""

import ctypes

import pytest
import torch

from paged_kv_cache_chunked_b200 import api
from paged_kv_cache_chunked_b200._lib import lib
from paged_kv_cache_chunked_b200.workloads import make_batch

from helpers import assert_close, gpu_pool_from, oracle_attention, recorded_ops

pytestmark = pytest.mark.gpu


def _noalloc_call(pool, b, dev):
    """The arguments of one no-allocation call (device copies of the batch),
    the output buffer, and the call itself as a function of the stream."""
    q = b["q"].to(dev)
    out = torch.full_like(q, float("nan"))
    tables = b["block_tables"].to(dev)
    ctx, qsl = b["context_lens"].to(dev), b["query_start_lens"].to(dev)

    def call(stream):
        return lib().pk_paged_attention_noalloc(
            pool.handle, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
            ctypes.c_void_p(tables.data_ptr()), tables.shape[1], ctypes.c_void_p(ctx.data_ptr()),
            ctypes.c_void_p(qsl.data_ptr()), ctx.shape[0], q.shape[0], q.shape[1],
            ctypes.c_float(b["scale"]), stream)
    return call, out, (q, tables, ctx, qsl)


def _noalloc(pool, b, dev):
    call, out, _keep = _noalloc_call(pool, b, dev)
    rc = call(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    torch.cuda.synchronize(dev)
    return rc, out


def _with_fresh_workspace(pool, b, dev):
    """pk_paged_attention with a newly zeroed workspace of its own."""
    n = ctypes.c_size_t()
    lib().pk_attention_workspace_size(pool.handle, b["context_lens"].shape[0], b["q"].shape[0],
                                      b["q"].shape[1], b["block_tables"].shape[1], ctypes.byref(n))
    ws = torch.zeros(n.value, dtype=torch.uint8, device=dev)
    q, tables = b["q"].to(dev), b["block_tables"].to(dev)
    ctx, qsl = b["context_lens"].to(dev), b["query_start_lens"].to(dev)
    out = torch.full_like(q, float("nan"))
    rc = lib().pk_paged_attention(
        pool.handle, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(tables.data_ptr()), tables.shape[1], ctypes.c_void_p(ctx.data_ptr()),
        ctypes.c_void_p(qsl.data_ptr()), ctx.shape[0], q.shape[0], q.shape[1],
        ctypes.c_float(b["scale"]), ctypes.c_void_p(ws.data_ptr()), n.value,
        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    torch.cuda.synchronize(dev)
    assert rc == 0, lib().pk_last_error()
    return out


def test_noalloc_matches_the_workspace_entry_point(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    batches = [
        make_batch([900, 33, 4000, 257], [1, 33, 1, 64], block_size=16, n_q_heads=32,
                   n_kv_heads=8, head_dim=128, dtype=torch.bfloat16, seed=41),
        make_batch([1200, 77], [1, 1], block_size=16, n_q_heads=32, n_kv_heads=8,
                   head_dim=128, dtype=torch.bfloat16, seed=42),
    ]
    for b in batches:      # two calls in a row through the shared scratch array
        pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
        ref = api.paged_attention(b["q"].to(cuda_dev), pool.k_pool, pool.v_pool,
                                  b["block_tables"].to(cuda_dev), b["context_lens"].to(cuda_dev),
                                  b["query_start_lens"].to(cuda_dev), b["scale"])
        rc, got = _noalloc(pool, b, cuda_dev)
        assert rc == 0, lib().pk_last_error()
        assert_close(got, ref, torch.bfloat16, "no-alloc vs workspace entry point")
        assert_close(got, oracle_attention(b), torch.bfloat16, "no-alloc vs oracle")
        assert pool.check_device_errors() == 0


# pools of different geometry in a row, each call compared with the workspace
# entry point on a fresh workspace and with the oracle:
#   - 2 kv heads then 8, with 16 and 10 q heads per kv head: decode rows on the
#     tile-streaming kernel, whose split-K arrival counters live in the array
#   - 600 sequences: two launch windows of 512
#   - 4 kv heads, head dim 256: block-streaming decode with its merge kernel
NOALLOC_CASES = [
    (dict(context_lens=[3000, 40, 1700], n_q_heads=32, n_kv_heads=2, head_dim=128), 51),
    (dict(context_lens=[2500, 900, 64, 1300], n_q_heads=80, n_kv_heads=8, head_dim=128), 52),
    (dict(context_lens=[1 + (i * 53) % 300 for i in range(600)], n_q_heads=8, n_kv_heads=2,
          head_dim=64), 53),
    (dict(context_lens=[5000, 20, 2100], n_q_heads=16, n_kv_heads=4, head_dim=256), 54),
]


def test_noalloc_across_pools_of_different_geometry(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    for kw, seed in NOALLOC_CASES:
        b = make_batch(kw["context_lens"], None, block_size=16, n_q_heads=kw["n_q_heads"],
                       n_kv_heads=kw["n_kv_heads"], head_dim=kw["head_dim"], dtype=torch.bfloat16,
                       seed=seed)
        pool = gpu_pool_from(b, kw["n_kv_heads"], kw["head_dim"], torch.bfloat16, cuda_dev)
        rc, got = _noalloc(pool, b, cuda_dev)
        assert rc == 0, lib().pk_last_error()
        what = f"Hkv {kw['n_kv_heads']}, {len(kw['context_lens'])} seqs"
        assert_close(got, _with_fresh_workspace(pool, b, cuda_dev), torch.bfloat16, what)
        assert_close(got, oracle_attention(b), torch.bfloat16, what + " vs oracle")
        assert pool.check_device_errors() == 0


def test_noalloc_clears_stale_counters(cuda_dev):
    # A call that gives up on a bounded wait can leave work-claim and split-K
    # counters set in the shared array.  Every call clears that region first:
    # its recorded work (recorded, not run) starts with one zero-fill on the
    # array, before any kernel.  Filling that region with non-zero bytes from
    # the host and then calling normally still gives the oracle's result.
    from cuda.bindings import runtime as rt
    torch.cuda.set_device(cuda_dev)
    b = make_batch([3000, 40, 1700, 800], None, block_size=16, n_q_heads=32, n_kv_heads=2,
                   head_dim=128, dtype=torch.bfloat16, seed=55)
    pool = gpu_pool_from(b, 2, 128, torch.bfloat16, cuda_dev)
    assert _noalloc(pool, b, cuda_dev)[0] == 0        # the array's address is known from here on
    call, out, _keep = _noalloc_call(pool, b, cuda_dev)
    s = torch.cuda.Stream(cuda_dev)
    torch.cuda.synchronize(cuda_dev)
    (err,) = rt.cudaStreamBeginCapture(rt.cudaStream_t(s.cuda_stream),
                                       rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == rt.cudaError_t.cudaSuccess
    try:
        rc = call(ctypes.c_void_p(s.cuda_stream))
    finally:
        err, graph = rt.cudaStreamEndCapture(rt.cudaStream_t(s.cuda_stream))
    assert rc == 0 and err == rt.cudaError_t.cudaSuccess
    _, _, n = rt.cudaGraphGetNodes(graph, 0)
    _, nodes, _ = rt.cudaGraphGetNodes(graph, n)
    _, _, n_roots = rt.cudaGraphGetRootNodes(graph, 0)
    _, roots, _ = rt.cudaGraphGetRootNodes(graph, n_roots)
    kinds = [rt.cudaGraphNodeGetType(x)[1] for x in nodes]
    memsets = [x for x, k in zip(nodes, kinds) if k == rt.cudaGraphNodeType.cudaGraphNodeTypeMemset]
    assert len(memsets) == 1 and n_roots == 1
    assert rt.cudaGraphNodeGetType(roots[0])[1] == rt.cudaGraphNodeType.cudaGraphNodeTypeMemset
    assert kinds.count(rt.cudaGraphNodeType.cudaGraphNodeTypeKernel) >= 1
    _, prm = rt.cudaGraphMemsetNodeGetParams(memsets[0])
    dst, nbytes = int(prm.dst), prm.width * prm.height * prm.elementSize
    assert prm.value == 0 and nbytes >= 512
    rt.cudaGraphDestroy(graph)
    # non-zero counters, then a normal call: on the tile-streaming decode kernel
    # (16 q heads per kv head), whose split heads are merged through those
    # counters, and on the block-streaming one with its merge kernel (48
    # sequences, 4 q heads per kv head), which must not depend on them
    b2 = make_batch([200 + (i * 97) % 2300 for i in range(48)], None, block_size=16, n_q_heads=32,
                    n_kv_heads=8, head_dim=128, dtype=torch.bfloat16, seed=57)
    pool2 = gpu_pool_from(b2, 8, 128, torch.bfloat16, cuda_dev)
    for pl, bb in ((pool, b), (pool2, b2)):
        (err,) = rt.cudaMemset(dst, 0x01, nbytes)
        assert err == rt.cudaError_t.cudaSuccess
        torch.cuda.synchronize(cuda_dev)
        rc, got = _noalloc(pl, bb, cuda_dev)
        assert rc == 0, lib().pk_last_error()
        assert_close(got, oracle_attention(bb), torch.bfloat16, "no-alloc after stale counters")
        assert pl.check_device_errors() == 0


def test_noalloc_with_no_sequences(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    b = make_batch([64], [1], block_size=16, n_q_heads=32, n_kv_heads=8, head_dim=128,
                   dtype=torch.bfloat16, seed=56, poison_unused=False)
    pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
    k0 = pool.k_pool.clone()
    qsl = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    null = ctypes.c_void_p(0)
    rc, n_ops = recorded_ops(cuda_dev, lambda st: lib().pk_paged_attention_noalloc(
        pool.handle, null, null, null, 1, null, ctypes.c_void_p(qsl.data_ptr()), 0, 0, 32,
        ctypes.c_float(0.125), st))
    assert (rc, n_ops) == (0, 0)
    torch.cuda.synchronize(cuda_dev)
    assert torch.equal(pool.k_pool, k0) and pool.check_device_errors() == 0


def test_noalloc_refuses_batches_beyond_its_scratch(cuda_dev):
    torch.cuda.set_device(cuda_dev)
    b = make_batch([64], [1], block_size=16, n_q_heads=32, n_kv_heads=8, head_dim=128,
                   dtype=torch.bfloat16, seed=43, poison_unused=False)
    pool = gpu_pool_from(b, 8, 128, torch.bfloat16, cuda_dev)
    need = ctypes.c_size_t()
    # 512 sequences with 16 q heads per kv head: split-K scratch past 32 MiB
    n_seqs, n_q_heads = 512, 128
    lib().pk_attention_workspace_size(pool.handle, n_seqs, n_seqs, n_q_heads, 4, ctypes.byref(need))
    assert need.value > 32 << 20
    dummy = ctypes.c_void_p(pool.k_pool.data_ptr())
    rc = lib().pk_paged_attention_noalloc(pool.handle, dummy, dummy, dummy, 4, dummy, dummy, n_seqs,
                                          n_seqs, n_q_heads, ctypes.c_float(1.0), None)
    assert rc == 6                             # PK_ERR_WORKSPACE, nothing launched
    assert b"scratch" in lib().pk_last_error()
