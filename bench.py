#!/usr/bin/env python
"""Benchmark of one step of the paged-KV hot path on B200.

A step is one decode iteration of the named workload: append each sequence's
new token's K/V into its block (paged_kv_append), then paged attention of
every sequence's query over its whole paged context (plan + attention +
split-K reduce kernels).  The workload has no forks, so the copy-on-write
block copy has no work in it.  Every step leaves the pool in the same state
(the appended rows are the values already stored at those slots), so all
steps are the same work.

Prints one JSON line.  `value` is the step's algorithmic bytes (KV read once
per sequence and kv head, Q and output, block tables, the append's reads and
writes) per second over all GPUs; `roofline` is the attention call alone.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload decode64_bf16|longdoc_bf16]
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_chunked_b200.workloads import WORKLOADS, workload_batch  # noqa: E402

METRIC = "paged decode attention KV GB/s (% of HBM peak) and tokens/s per scheduler step"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "paged_kv_cache_chunked_b200", "csrc")
# the source of each workload's dominant kernel (the traffic record is valid for that source only)
KERNEL_SRC = {"chunk512_bf16": os.path.join(CSRC, "attention_chunk_umma.cu"),
              "append_copy": os.path.join(CSRC, "kv_copy.cu")}
DECODE_SRC = os.path.join(CSRC, "attention_decode_blocks.cu")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="decode64_bf16",
                   choices=["decode64_bf16", "longdoc_bf16", "chunk512_bf16", "trace", "trace_swap",
                            "trace_prefix", "trace_prefix_nocache", "trace_hybrid", "policy", "fork",
                            "fork1028", "append_copy"])
    p.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--profile-run", action="store_true",
                   help="timed steps only: no clock window, no e2e leg, no CPU baseline")
    return p.parse_args()


# ---------------------------------------------------------------- work accounting
def step_bytes(batch):
    """Algorithmic bytes of one step: attention and append separately."""
    q = batch["q"]
    T, Hq, d = q.shape
    _, Hkv, bs, _ = batch["k_pool"].shape
    elt = q.element_size()
    ctx = batch["context_lens"].to(torch.int64)
    kv = int(ctx.sum()) * Hkv * d * elt * 2
    tables = int(((ctx + bs - 1) // bs).sum()) * 4
    attn = kv + 2 * T * Hq * d * elt + tables
    append = 2 * (2 * T * Hkv * d * elt) + 8 * T
    return attn, append, kv


def last_token_slots(batch):
    """Slots of every sequence's query tokens (its last q_b positions)."""
    bs = batch["block_size"]
    ctx = batch["context_lens"].to(torch.int64)
    qsl = batch["query_start_lens"].to(torch.int64)
    tables = batch["block_tables"].to(torch.int64)
    slots = []
    for b in range(ctx.shape[0]):
        qn = int(qsl[b + 1] - qsl[b])
        pos = torch.arange(int(ctx[b]) - qn, int(ctx[b]))
        slots.append(tables[b, pos // bs] * bs + pos % bs)
    return torch.cat(slots)


def attention_flops(batch):
    """4 * Hq * d per visible (query row, key) pair (QK^T and PV, 2 flops per MAC)."""
    T, Hq, d = batch["q"].shape
    ctx = batch["context_lens"].to(torch.int64).tolist()
    qsl = batch["query_start_lens"].to(torch.int64).tolist()
    keys = 0
    for b, c in enumerate(ctx):
        qn = qsl[b + 1] - qsl[b]
        keys += qn * (c - qn) + qn * (qn + 1) // 2
    return 4 * Hq * d * keys


def new_token_kv(batch, slots):
    bs = batch["block_size"]
    blk, off = slots // bs, slots % bs
    return batch["k_pool"][blk, :, off].contiguous(), batch["v_pool"][blk, :, off].contiguous()


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(workload):
    """DRAM bytes per attention call from the committed ncu summary, if it was
    taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    with open(KERNEL_SRC.get(workload, DECODE_SRC), "rb") as f:
        src_hash = hashlib.sha256(f.read()).hexdigest()[:16]
    entry = rec.get(workload)
    if not entry or entry.get("kernel_sha256_16") != src_hash:
        return None
    return entry.get("dram_bytes_per_call")


# ---------------------------------------------------------------- CPU / oracle arm
def oracle_step_seconds(batch, budget_s, min_runs=1):
    """The oracle's attention over the whole workload batch, repeated for about
    budget_s seconds; returns (seconds per run, runs, threads)."""
    import oracle
    runs, t0 = 0, time.perf_counter()
    while runs < min_runs or time.perf_counter() - t0 < budget_s:
        oracle.paged_attention(batch["q"], batch["k_pool"], batch["v_pool"], batch["block_tables"],
                               batch["context_lens"], batch["query_start_lens"], batch["scale"])
        runs += 1
    return (time.perf_counter() - t0) / runs, runs, oracle.num_threads()


def subset_batch(batch, n):
    """The first n sequences of a batch (same pools)."""
    qsl = batch["query_start_lens"]
    t1 = int(qsl[n])
    sub = dict(batch)
    sub["q"] = batch["q"][:t1]
    sub["block_tables"] = batch["block_tables"][:n]
    sub["context_lens"] = batch["context_lens"][:n]
    sub["query_start_lens"] = qsl[:n + 1]
    return sub


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores (rank 0 only).  Each step is
    the oracle append plus float64 attention over a leading subset of the
    workload's sequences, sized so that the whole run stays near two
    minutes."""
    if rank != 0:
        return
    import oracle
    if args.workload == "append_copy":
        run_reference_kvops(args, world)
        return
    batch = workload_batch(args.workload, poison_unused=False)
    slots = last_token_slots(batch)
    k_new, v_new = new_token_kv(batch, slots)
    kp, vp = batch["k_pool"].clone(), batch["v_pool"].clone()

    def step(b, n):
        oracle.kv_append(kp, vp, k_new[:n], v_new[:n], slots[:n])
        oracle.paged_attention(b["q"], kp, vp, b["block_tables"], b["context_lens"],
                               b["query_start_lens"], b["scale"])

    B = batch["context_lens"].shape[0]
    t0 = time.perf_counter()
    step(batch, B)
    t_full = time.perf_counter() - t0
    frac = min(1.0, 120.0 / max(1, args.steps + args.warmup) / t_full)
    ctx = batch["context_lens"].to(torch.int64)
    cum = torch.cumsum(ctx, 0)
    n = int(min(B, max(1, int((cum < frac * int(ctx.sum())).sum()) + 1)))
    sample = subset_batch(batch, n)
    attn_b, app_b, _ = step_bytes(sample)
    for _ in range(args.warmup):
        step(sample, n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(sample, n)
    dt = (time.perf_counter() - t0) / args.steps
    value = (attn_b + app_b) / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(args.workload, batch, "oracle on host cores: L2 not applicable"),
        "tokens_per_s": n / dt,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"each step: oracle append + float64 attention of the first "
                                   f"{n} of {B} sequences of {args.workload} "
                                   f"({int(sample['context_lens'].sum())} context tokens)"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_kvops(args, world):
    """The oracle's append + block copy on the host, each step 1/16 of the
    append_copy workload (4,096 tokens, 128 block pairs)."""
    import oracle
    w = KVOPS
    slots, k, v, pairs = kvops_inputs()
    n, m = w["tokens"] // 16, w["pairs"] // 16
    kp = torch.zeros(w["num_blocks"], w["n_kv_heads"], w["block_size"], w["head_dim"], dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    app_b, copy_b = kvops_bytes()

    def step():
        oracle.kv_append(kp, vp, k[:n], v[:n], slots[:n])
        oracle.block_copy(kp, vp, pairs[:m])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = (app_b + copy_b) / 16 / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "append_copy", **w, "l2": "oracle on host cores: L2 not applicable"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: oracle kv_append of {n} tokens + block_copy of {m} blocks"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def roofline_entry(workload, attn_b, flops, avg_ms, gbs, tflops, hbm_peak, hbm_kind):
    """The attention call's roofline: HBM for decode (about 4 flop/byte at GQA 4),
    the tensor pipe for prefill chunks (a dense contraction)."""
    kern = ("paged_attention call: tcgen05 chunk kernel (S and O accumulated in tensor memory)"
            if workload == "chunk512_bf16" else
            "paged_attention call: block-streaming decode kernel + split-K merge kernel")
    common = {"kernel": kern,
              "algorithmic_bytes": attn_b, "algorithmic_flops": flops, "avg_ms": avg_ms,
              "traffic": kernel_traffic(workload)}
    if workload == "chunk512_bf16":
        peak, kind = measured_tensor_peak()
        return dict(common, bound="tensor", achieved=tflops, peak=peak, unit="TFLOP/s",
                    frac=tflops / peak,
                    peak_source=f"{kind} (MEASURED_PEAKS.json bf16_tflops, burst)")
    return dict(common, bound="hbm", achieved=gbs, peak=hbm_peak, unit="GB/s",
                frac=gbs / hbm_peak,
                peak_source=f"{hbm_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if hbm_kind == "measured" else "fallback 6.65 TB/s")


def workload_config(name, batch, l2_note):
    w = WORKLOADS[name]
    ctx = batch["context_lens"]
    return {"workload": name, "num_seqs": int(ctx.shape[0]), "context_tokens": int(ctx.sum()),
            "n_q_heads": w["n_q_heads"], "n_kv_heads": w["n_kv_heads"], "head_dim": w["head_dim"],
            "block_size": w["block_size"], "num_blocks": int(batch["k_pool"].shape[0]),
            "seed": w["seed"], "l2": l2_note, "parallelism": "replicas"}


# ---------------------------------------------------------------- our arm
def attention_call_ms(call, stream, n):
    """Device ms of each of n calls, every call between two CUDA events on the
    stream it is launched on (after 3 untimed calls)."""
    for _ in range(3):
        call()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def workload_roofline(name, device, n_calls):
    """Roofline of one pk_paged_attention call on another decode workload (the
    long-document one rides along with the default line)."""
    from paged_kv_cache_chunked_b200 import api
    batch = workload_batch(name, poison_unused=False)
    attn_b, _, kv_b = step_bytes(batch)
    N, Hkv, bs, d = batch["k_pool"].shape
    pool = api.kv_pool_create(N, bs, Hkv, d, torch.bfloat16, device)
    pool.k_pool.copy_(batch["k_pool"])
    pool.v_pool.copy_(batch["v_pool"])
    dq, dt_ = batch["q"].to(device), batch["block_tables"].to(device)
    dctx, dqsl = batch["context_lens"].to(device), batch["query_start_lens"].to(device)
    out = torch.empty_like(dq)
    stream = torch.cuda.current_stream(device)
    ms = attention_call_ms(lambda: api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl,
                                                       batch["scale"], out=out), stream, n_calls)
    assert pool.check_device_errors() == 0
    peak, kind = measured_peak()
    avg = statistics.mean(ms)
    gbs = attn_b / (avg * 1e-3) / 1e9
    r = roofline_entry(name, attn_b, attention_flops(batch), avg, gbs, None, peak, kind)
    r.update(calls=n_calls, config=workload_config(name, batch, f"no flush: {kv_b / 1e6:.0f} MB of KV "
                                                                f"per call, more than the 126 MB L2"))
    del pool
    torch.cuda.empty_cache()
    return r


def run_ours(args, rank, world, device):
    from paged_kv_cache_chunked_b200 import api

    batch = workload_batch(args.workload, poison_unused=False)
    attn_b, app_b, kv_b = step_bytes(batch)
    T, Hq, d = batch["q"].shape
    N, Hkv, bs, _ = batch["k_pool"].shape
    slots = last_token_slots(batch)
    k_new, v_new = new_token_kv(batch, slots)

    pool = api.kv_pool_create(N, bs, Hkv, d, torch.bfloat16, device)
    pool.k_pool.copy_(batch["k_pool"])
    pool.v_pool.copy_(batch["v_pool"])
    dq = batch["q"].to(device)
    dt_ = batch["block_tables"].to(device)
    dctx = batch["context_lens"].to(device)
    dqsl = batch["query_start_lens"].to(device)
    dslots = slots.to(device)
    dk, dv = k_new.to(device), v_new.to(device)
    out = torch.empty_like(dq)
    stream = torch.cuda.current_stream(device)

    def step():
        api.paged_kv_append(dk, dv, dslots, pool=pool)
        api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"], out=out)

    def attention_only():
        api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"], out=out)

    # append, then per window of 512 sequences: for a batch of decodes only
    # (groups of <= 8 q heads) the block-streaming kernel and its merge kernel,
    # else the chunk kernel (when chunks are present) and the tile-streaming
    # decode kernel; the general kernel is one launch
    tc = pool.dtype == torch.bfloat16 and d in (64, 128, 256) and bs % 8 == 0
    B = batch["context_lens"].shape[0]
    windows = (B + 511) // 512
    blocks_path = tc and T == B and Hq // Hkv <= 8
    per_window = 2 if blocks_path else (2 if T > B or Hq // Hkv > 16 else 1)
    launches_per_step = 1 + (windows * per_window if tc else 1)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    assert pool.check_device_errors() == 0

    dist = world > 1
    if dist:
        import torch.distributed as tdist
    clocks = ClockSampler(device.index if device.index is not None else 0)
    if not args.profile_run:
        clocks.start()
        time.sleep(0.3)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        tdist.barrier()
    torch.cuda.synchronize(device)
    start.record(stream)
    for i in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    if dist:
        tdist.barrier()
    total_ms = start.elapsed_time(end)
    # the attention call alone, for its roofline: a separate pass, so that no
    # event sits between the append and the attention of a timed step (the
    # attention kernels start as programmatic dependents of the append)
    attn_ms = attention_call_ms(attention_only, stream, max(args.steps, 50))
    # a long enough window for the clock sampler to see the load
    t_extra = time.perf_counter()
    while not args.profile_run and time.perf_counter() - t_extra < 1.0:
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)
    clk = clocks.stop() if not args.profile_run else {"sm_mhz": None, "reasons": ["not sampled"]}
    assert pool.check_device_errors() == 0

    if dist:
        t = torch.tensor([total_ms], device=device)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    value = world * (attn_b + app_b) / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API: pinned host inputs in, output back out
    e2e = None
    if not args.no_e2e and not args.profile_run:
        h_q = batch["q"].pin_memory()
        h_k, h_v = k_new.pin_memory(), v_new.pin_memory()
        h_slots = slots.pin_memory()
        h_t = batch["block_tables"].pin_memory()
        h_ctx = batch["context_lens"].pin_memory()
        h_qsl = batch["query_start_lens"].pin_memory()
        h_out = torch.empty_like(batch["q"]).pin_memory()
        bufs = [torch.empty_like(x, device=device) for x in (h_q, h_k, h_v, h_slots, h_t, h_ctx, h_qsl)]
        h2d = sum(x.numel() * x.element_size() for x in (h_q, h_k, h_v, h_slots, h_t, h_ctx, h_qsl))
        d2h = h_out.numel() * h_out.element_size()

        def e2e_step():
            for dst, src in zip(bufs, (h_q, h_k, h_v, h_slots, h_t, h_ctx, h_qsl)):
                dst.copy_(src, non_blocking=True)
            api.paged_kv_append(bufs[1], bufs[2], bufs[3], pool=pool)
            o = api.paged_attention(bufs[0], pool.k_pool, pool.v_pool, bufs[4], bufs[5], bufs[6],
                                    batch["scale"], out=out)
            h_out.copy_(o, non_blocking=True)

        for _ in range(3):
            e2e_step()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            tdist.barrier()
        torch.cuda.synchronize(device)
        s2.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(device)
        e_ms = s2.elapsed_time(e2)
        if dist:
            t = torch.tensor([e_ms], device=device)
            tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
            e_ms = float(t.item())
        e_ms /= args.steps
        e2e = {"value": world * (attn_b + app_b) / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        assert torch.isfinite(h_out.float()).all()

    if rank != 0:
        return
    peak, peak_kind = measured_peak()
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = attn_b / (attn_avg_ms * 1e-3) / 1e9
    flops = attention_flops(batch)
    tflops = flops / (attn_avg_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args.workload, batch,
                                  f"no flush: the step reads {kv_b / 1e6:.0f} MB of KV, "
                                  f"more than the 126 MB L2"),
        "pct_hbm": 100.0 * value / world / peak,
        "tokens_per_s": world * T / (ms_per_step * 1e-3),
        "roofline": roofline_entry(args.workload, attn_b, flops, attn_avg_ms, achieved, tflops,
                                   peak, peak_kind),
        "attention_tflops": tflops,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": dict(clk, window="the timed region plus 1 s of the same steps right after it"),
        "attention_timing": f"{len(attn_ms)} attention calls, each between CUDA events, in a pass "
                            f"after the timed steps",
    }
    if e2e:
        line["e2e"] = e2e
    if args.workload == "decode64_bf16" and not args.profile_run and world == 1:
        clocks2 = ClockSampler(device.index if device.index is not None else 0)
        clocks2.start()
        time.sleep(0.3)
        extra = workload_roofline("longdoc_bf16", device, max(50, min(args.steps, 1000)))
        extra["clocks"] = clocks2.stop()
        line["extra_rooflines"] = {"longdoc_bf16": extra}
    if world == 1 and args.cpu_baseline_seconds > 0 and not args.profile_run:
        sec, runs, threads = oracle_step_seconds(batch, args.cpu_baseline_seconds)
        line["cpu_baseline"] = {"value": attn_b / sec / 1e9, "unit": "GB/s", "cores": threads,
                                "kind": "oracle",
                                "sample": f"float64 oracle attention over the whole {args.workload} "
                                          f"batch (attention bytes only), {runs} runs"}
    print(json.dumps(line), flush=True)


# KV append and block copy alone, at sizes well above L2: 65,536 new tokens
# written to distinct random slots of a decode-64-shaped pool (8 kv heads, head
# dim 128, 16-token blocks, bf16), then 2,048 whole blocks copied (the
# copy-on-write step of a fork).
KVOPS = dict(num_blocks=9594, n_kv_heads=8, block_size=16, head_dim=128, tokens=65536, pairs=2048,
             seed=1007)


def kvops_inputs():
    w = KVOPS
    g = torch.Generator().manual_seed(w["seed"])
    N, H, bs, d = w["num_blocks"], w["n_kv_heads"], w["block_size"], w["head_dim"]
    T = w["tokens"]
    slots = torch.randperm(N * bs, generator=g)[:T]
    k = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    v = torch.randn(T, H, d, generator=g).to(torch.bfloat16)
    perm = torch.randperm(N, generator=g)
    pairs = torch.stack([perm[:w["pairs"]], perm[w["pairs"]:2 * w["pairs"]]], 1).to(torch.int32)
    return slots, k, v, pairs


def kvops_bytes():
    w = KVOPS
    tok = w["n_kv_heads"] * w["head_dim"] * 2  # one token's K (or V) row set, bf16
    append = 2 * (2 * w["tokens"] * tok) + 8 * w["tokens"]  # read new K, V; write them; slots
    blk = w["n_kv_heads"] * w["block_size"] * w["head_dim"] * 2 * 2  # K + V of one block
    copy = 2 * w["pairs"] * blk + 8 * w["pairs"]  # read + write each block; the pairs
    return append, copy


def run_kvops(args, rank, world, device):
    from paged_kv_cache_chunked_b200 import api
    w = KVOPS
    slots, k, v, pairs = kvops_inputs()
    app_b, copy_b = kvops_bytes()
    pool = api.kv_pool_create(w["num_blocks"], w["block_size"], w["n_kv_heads"], w["head_dim"],
                              torch.bfloat16, device)
    ds, dk, dv, dp = slots.to(device), k.to(device), v.to(device), pairs.to(device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        api.paged_kv_append(dk, dv, ds, pool=pool)
        if ev is not None:
            ev[1].record(stream)
        api.block_copy(dp, pool=pool)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(device)
    assert pool.check_device_errors() == 0
    clocks = ClockSampler(device.index if device.index is not None else 0)
    if not args.profile_run:
        clocks.start()
        time.sleep(0.3)
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
    torch.cuda.synchronize(device)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(device)
    total_ms = start.elapsed_time(end)
    if world > 1:
        t = torch.tensor([total_ms], device=device)
        tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
        total_ms = float(t.item())
    t_extra = time.perf_counter()
    while not args.profile_run and time.perf_counter() - t_extra < 1.0:
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)
    clk = clocks.stop() if not args.profile_run else {"sm_mhz": None, "reasons": ["not sampled"]}
    assert pool.check_device_errors() == 0
    app_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in evs)
    copy_ms = statistics.mean(b.elapsed_time(c) for _, b, c in evs)
    ms_per_step = total_ms / args.steps
    value = world * (app_b + copy_b) / (ms_per_step * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e and not args.profile_run:
        hs, hk, hv, hp = (x.pin_memory() for x in (slots, k, v, pairs))
        h_out = torch.empty(w["n_kv_heads"], w["block_size"], w["head_dim"], dtype=torch.bfloat16).pin_memory()
        bufs = [torch.empty_like(x, device=device) for x in (hs, hk, hv, hp)]
        h2d = sum(x.numel() * x.element_size() for x in (hs, hk, hv, hp))
        d2h = h_out.numel() * h_out.element_size()
        dst0 = int(pairs[0, 1])

        def e2e_step():
            for dst, src in zip(bufs, (hs, hk, hv, hp)):
                dst.copy_(src, non_blocking=True)
            api.paged_kv_append(bufs[1], bufs[2], bufs[0], pool=pool)
            api.block_copy(bufs[3], pool=pool)
            h_out.copy_(pool.k_pool[dst0], non_blocking=True)  # one copied block back

        for _ in range(3):
            e2e_step()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(device)
        s2.record(stream)
        n_e2e = max(1, min(args.steps, 200))
        for _ in range(n_e2e):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(device)
        e_ms = s2.elapsed_time(e2) / n_e2e
        e2e = {"value": world * (app_b + copy_b) / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if rank != 0:
        return
    peak, peak_kind = measured_peak()
    ach = app_b / (app_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "append_copy", **{k_: v_ for k_, v_ in w.items()},
                   "l2": "no flush: each step moves 0.8 GB, more than the 126 MB L2",
                   "parallelism": "replicas"},
        "pct_hbm": 100.0 * value / world / peak,
        "append_gbs": ach, "copy_gbs": copy_b / (copy_ms * 1e-3) / 1e9,
        "roofline": {"kernel": "kv_append (paged_kv_append of 65,536 tokens)", "bound": "hbm",
                     "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                     "algorithmic_bytes": app_b, "avg_ms": app_ms, "traffic": kernel_traffic("append_copy"),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"},
        "gpu_launches": 2 * args.steps,
        "clocks": dict(clk, window="the timed region plus 1 s of the same steps right after it"),
    }
    if e2e:
        line["e2e"] = e2e
    if world == 1 and args.cpu_baseline_seconds > 0 and not args.profile_run:
        import oracle
        n = 4096  # bounded sample: 1/16 of the tokens, 1/16 of the pairs
        kp = torch.zeros(w["num_blocks"], w["n_kv_heads"], w["block_size"], w["head_dim"],
                         dtype=torch.bfloat16)
        vp = torch.zeros_like(kp)
        runs, t0 = 0, time.perf_counter()
        while runs < 1 or time.perf_counter() - t0 < args.cpu_baseline_seconds:
            oracle.kv_append(kp, vp, k[:n], v[:n], slots[:n])
            oracle.block_copy(kp, vp, pairs[:w["pairs"] // 16])
            runs += 1
        sec = (time.perf_counter() - t0) / runs
        line["cpu_baseline"] = {"value": (app_b + copy_b) / 16 / sec / 1e9, "unit": "GB/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"oracle kv_append of {n} tokens + block_copy of "
                                          f"{w['pairs'] // 16} blocks (1/16 of a step), {runs} runs"}
    print(json.dumps(line), flush=True)


def run_serving(args, rank, world, device):
    """Scheduler-driven workloads: the continuous-batching trace (300
    iterations, Poisson arrivals, chunked prefill, preemption) or n-sample
    forks with copy-on-write.  Reports tokens/s per scheduler step over the
    GPU time of copy + append + attention, and KV GB/s."""
    from paged_kv_cache_chunked_b200.drivers import ForkRunner, TraceRunner
    peak, peak_kind = measured_peak()
    kv_tok = 8 * 128 * 2 * 2          # K+V bytes per token per layer (8 kv heads, d 128, bf16)
    recs = []
    if args.workload.startswith("trace"):
        # trace_swap: preempted requests' blocks go to a pinned host pool of
        # 8,192 blocks and back instead of being recomputed.  trace_prefix:
        # every request starts with one of four shared system prompts (1,024,
        # 512, 2,048 or 256 tokens) whose blocks are shared through the prefix
        # cache; trace_prefix_nocache runs the same trace without the cache.
        from paged_kv_cache_chunked_b200.workloads import prefix_trace_requests
        # trace_hybrid: the same memory as trace's 8,192 blocks split into two
        # pools, 64 per-sequence state slots of 32 blocks' worth each and 6,144
        # KV blocks (a hybrid model's fixed-size state beside its paged KV)
        swap = args.workload == "trace_swap"
        prefix = args.workload.startswith("trace_prefix")
        hybrid = args.workload == "trace_hybrid"
        r = TraceRunner(device, preempt="swap" if swap else "recompute", num_host_blocks=8192 if swap else 0,
                        trace=prefix_trace_requests() if prefix else None,
                        prefix_cache=args.workload == "trace_prefix",
                        num_blocks=6144 if hybrid else 8192, state_slots=64 if hybrid else 0)
        while r.sched.step_no < 300 and (r.pending or r.sched.has_work()):
            rec = r.step()
            if rec is not None:
                recs.append(rec)
        skip = min(args.warmup, len(recs) // 2)
        recs = recs[skip:]
        cfg = {"workload": args.workload, "steps_run": len(recs) + skip, "warmup_steps": skip,
               "num_blocks": r.bm.num_blocks, "block_size": 16, "n_q_heads": 32, "n_kv_heads": 8,
               "head_dim": 128, "token_budget": 4096, "max_chunk": 512,
               "preempt": r.sched.preempt_mode,
               "preemptions": r.sched.metrics["preemptions"], "rejected": r.rejected,
               "finished": len(r.sched.finished)}
        if hybrid:
            cfg.update(state_slots=64, state_slot_blocks_worth=32,
                       max_running=max(x.num_seqs for x in recs))
        if prefix:
            st = r.bm.stats()
            cfg.update(trace="prefix_trace_requests(seed 1007): system prompts 1024/512/2048/256, user "
                             "median 256", prefix_cache=r.sched.prefix_cache,
                       prefix_lookups_blocks=st["prefix_lookups"], prefix_hits_blocks=st["prefix_hits"],
                       prefix_hit_rate=st["prefix_hits"] / max(st["prefix_lookups"], 1),
                       prefix_hit_tokens=r.sched.metrics["prefix_hit_tokens"],
                       gpu_ms_timed_steps=sum(x.gpu_ms for x in recs))
        if swap:
            cfg.update(host_blocks=8192, swaps_out=r.sched.metrics["swaps_out"],
                       swaps_in=r.sched.metrics["swaps_in"],
                       swapped_blocks_timed=sum(x.swap_blocks for x in recs))
        ms = [x.gpu_ms for x in recs]
        toks = [x.tokens for x in recs]
        useful = sum(x.new_tokens for x in recs)
        kvb = [x.context_tokens * kv_tok for x in recs]
        copies = sum(x.copies for x in recs)
    else:
        plen = 1028 if args.workload == "fork1028" else 1024
        r = ForkRunner(device, prompt_len=plen)
        r.prefill()
        for _ in range(min(args.warmup, 8)):
            r.decode_step()
        ms, toks, kvb, copies = [], [], [], 0
        steps = min(args.steps, r.decode_steps - min(args.warmup, 8))
        for _ in range(steps):
            before_unique = r.unique_blocks()
            t, c = r.decode_step()
            ms.append(t)
            toks.append(len(r.seqs))
            kvb.append(before_unique * 16 * kv_tok)     # unique (physical) blocks read
            copies += c
        cfg = {"workload": args.workload, "prompts": 64, "prompt_len": plen, "samples": 4,
               "block_size": 16, "n_q_heads": 32, "n_kv_heads": 8, "head_dim": 128,
               "decode_steps_timed": steps, "unique_blocks": r.unique_blocks(),
               "clone_blocks": r.clone_blocks(), "copies": copies}
        useful = sum(toks)
    tot_ms = sum(ms)
    per_step = sorted(t / (m * 1e-3) for t, m in zip(toks, ms))
    pct = lambda q: per_step[min(len(per_step) - 1, int(q * len(per_step)))]
    line = {"metric": METRIC, "value": sum(toks) / (tot_ms * 1e-3), "unit": "tokens/s",
            "n_gpus": world, "steps": len(ms), "warmup": args.warmup, "ms_per_step": tot_ms / len(ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg,
            "tokens_per_step_s": {"p10": pct(0.1), "p50": pct(0.5), "p90": pct(0.9)},
            # positions stored for the first time: recomputed prefill tokens excluded
            "useful_tokens_per_s": useful / (tot_ms * 1e-3),
            "kv_gbs": sum(kvb) / (tot_ms * 1e-3) / 1e9,
            "pct_hbm": 100 * sum(kvb) / (tot_ms * 1e-3) / 1e9 / peak,
            "timing": "per-step CUDA events around swaps + copy + append + attention; host scheduling excluded"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_policy(args, rank, world, device):
    """Scheduler policy study ["Batching and PagedAttention", "Scheduling is a
    policy" and "Static batching"; 7.8 PagedAttention & continuous batching,
    "01 Concept": queue delay, time to first token, inter-token latency by
    request class]: one serving trace (about one arrival a step for 300 steps,
    333 requests) run to completion under continuous batching with token
    budgets of 1,024, 2,048, 4,096 and 8,192 per step, and under static
    batching (batches of 64, budget 4,096).  Latencies are in scheduler steps
    and in GPU ms (per-step CUDA events, summed); value is the tokens/s of the
    4,096 continuous configuration."""
    from paged_kv_cache_chunked_b200.drivers import TraceRunner
    from paged_kv_cache_chunked_b200.scheduler import summary
    from paged_kv_cache_chunked_b200.workloads import trace_requests
    trace = trace_requests(n_steps=300, arrivals_per_step=1.0, seed=1004)
    configs = [("continuous_1024", dict(token_budget=1024)), ("continuous_2048", dict(token_budget=2048)),
               ("continuous_4096", dict(token_budget=4096)), ("continuous_8192", dict(token_budget=8192)),
               ("static64_4096", dict(token_budget=4096, static_batch=64))]
    pick = lambda st, k: None if st is None else {q: st[q] for q in ("p50", "p90")} if k else st
    study = {}
    for name, kw in configs:
        r = TraceRunner(device, trace=trace, **kw)
        while r.pending or r.sched.has_work():
            r.step()
        ms = r.step_ms()
        tot = sum(ms)
        summ = summary(r.sched.finished, ms)
        study[name] = {
            "steps": r.sched.step_no, "finished": len(r.sched.finished), "gpu_ms": tot,
            "tokens_per_s": sum(x.tokens for x in r.records) / (tot * 1e-3),
            "useful_tokens_per_s": sum(x.new_tokens for x in r.records) / (tot * 1e-3),
            "preemptions": r.sched.metrics["preemptions"],
            "by_class": {cls: {"requests": v["requests"], "queue_delay_steps": pick(v["queue_delay"], 1),
                               "ttft_steps": pick(v["ttft"], 1), "ttft_ms": pick(v["ttft_ms"], 1),
                               "itl_ms": pick(v["itl_ms"], 1)}
                         for cls, v in summ.items()}}
    base = study["continuous_4096"]
    line = {"metric": METRIC, "value": base["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
            "steps": base["steps"], "warmup": 0, "ms_per_step": base["gpu_ms"] / base["steps"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "policy", "trace": "trace_requests(arrivals 1.0/step, 300 steps, seed 1004)",
                       "requests": len(trace), "num_blocks": 8192, "block_size": 16, "max_chunk": 512},
            "study": study,
            "timing": "per-step CUDA events around copy + append + attention, summed; host scheduling excluded"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=device)
    try:
        if args.workload == "policy":
            run_policy(args, rank, world, device)
        elif args.workload.startswith("trace") or args.workload in ("fork", "fork1028"):
            run_serving(args, rank, world, device)
        elif args.workload == "append_copy":
            run_kvops(args, rank, world, device)
        else:
            run_ours(args, rank, world, device)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    main()
