"""Shared test helpers: moving a seeded batch onto the GPU pool and comparing
the CUDA path with the oracle."""

import math

import torch

import oracle
from paged_kv_cache_chunked_b200 import api

TOL = {torch.bfloat16: (2e-2, 2e-2), torch.float32: (1e-4, 1e-4)}


def assert_close(got, ref, dtype, what=""):
    """|got - ref| <= atol + rtol * |ref| element by element (the allclose
    reading of the stated absolute and relative bounds)."""
    atol, rtol = TOL[dtype]
    got = got.detach().to("cpu", torch.float64)
    ref = ref.detach().to("cpu", torch.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{what}: non-finite output"
    err = (got - ref).abs()
    bound = atol + rtol * ref.abs()
    bad = err > bound
    if bad.any():
        i = int(bad.flatten().nonzero()[0])
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first at flat "
                             f"{i}: got {got.flatten()[i]:.6g} ref {ref.flatten()[i]:.6g}; "
                             f"max abs err {err.max():.3g}")
    return float(err.max())


def gpu_pool_from(batch, n_kv_heads, head_dim, dtype, device):
    """A KVPool whose contents are the batch's pools."""
    N = batch["k_pool"].shape[0]
    pool = api.kv_pool_create(N, batch["block_size"], n_kv_heads, head_dim, dtype, device)
    pool.k_pool.copy_(batch["k_pool"])
    pool.v_pool.copy_(batch["v_pool"])
    return pool


def run_gpu_attention(batch, pool, device):
    q = batch["q"].to(device)
    out = api.paged_attention(q, pool.k_pool, pool.v_pool, batch["block_tables"].to(device),
                              batch["context_lens"].to(device),
                              batch["query_start_lens"].to(device), batch["scale"])
    torch.cuda.synchronize(device)
    return out


def oracle_attention(batch):
    return oracle.paged_attention(batch["q"], batch["k_pool"], batch["v_pool"],
                                  batch["block_tables"], batch["context_lens"],
                                  batch["query_start_lens"], batch["scale"])


def sample_rows(num_tokens, n_q_heads, n, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.randint(0, num_tokens, (n,), generator=g)
    h = torch.randint(0, n_q_heads, (n,), generator=g)
    rows = torch.stack([t, h], 1)
    # always include the first and last rows
    extra = torch.tensor([[0, 0], [num_tokens - 1, n_q_heads - 1]])
    return torch.cat([rows, extra]).tolist()


def scale_of(head_dim):
    return 1.0 / math.sqrt(head_dim)


def recorded_ops(device, call):
    """Number of operations (kernels, copies, memsets) that call(stream)
    queues on a fresh stream: the stream is put in capture mode, so the work
    is recorded in a CUDA graph, counted and dropped, never run."""
    import ctypes

    from cuda.bindings import runtime as rt
    s = torch.cuda.Stream(device)
    torch.cuda.synchronize(device)
    (err,) = rt.cudaStreamBeginCapture(rt.cudaStream_t(s.cuda_stream),
                                       rt.cudaStreamCaptureMode.cudaStreamCaptureModeRelaxed)
    assert err == rt.cudaError_t.cudaSuccess, err
    try:
        rc = call(ctypes.c_void_p(s.cuda_stream))
    finally:
        err, graph = rt.cudaStreamEndCapture(rt.cudaStream_t(s.cuda_stream))
    assert err == rt.cudaError_t.cudaSuccess, err
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    assert err == rt.cudaError_t.cudaSuccess, err
    rt.cudaGraphDestroy(graph)
    return rc, n
