#!/usr/bin/env python
"""Benchmark of one step of the paged-KV hot path on B200.

A step is one decode iteration of the named workload in one call
(paged_attention_append): each sequence's new token's K/V stored at its
position through the block table, then paged attention of every sequence's
query over its whole paged context (the block-streaming kernel stores the new
rows itself; its split-K merge kernel follows).  The same step as two calls
(paged_kv_append with slots, then paged_attention) is timed beside it.  The
workload has no forks, so the copy-on-write block copy has no work in it.
Every step leaves the pool in the same state (the appended rows are the values
already stored at those slots), so all steps are the same work.

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
# the sources of each workload's dominant kernel, its local headers included
# (the traffic record is valid for those sources only)
_TC = ["tc_common.cuh", "pk_internal.h"]
KERNEL_SRC = {"chunk512_bf16": ["attention_chunk_umma.cu", "umma_common.cuh"] + _TC,
              "chunk512_d256_bf16": ["attention_chunk_umma256.cu", "umma_common.cuh"] + _TC,
              "append_copy": ["kv_copy.cu", "pk_internal.h"]}
DECODE_SRC = ["attention_decode_blocks.cu"] + _TC


def kernel_source_hash(workload):
    """sha256 (first 16 hex digits) of the dominant kernel's sources, in order."""
    h = hashlib.sha256()
    for name in KERNEL_SRC.get(workload, DECODE_SRC):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="decode64_bf16",
                   choices=["decode64_bf16", "longdoc_bf16", "chunk512_bf16", "chunk512_d256_bf16", "mixed_bf16",
                            "trace", "trace_swap",
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


# ---------------------------------------------------------------- ranks
def max_over_ranks(ms, device):
    """The slowest rank's time: replicas run the same work, and the job is done
    when the last one is (the one collective of a multi-GPU run)."""
    import torch.distributed as tdist
    if not tdist.is_available() or not tdist.is_initialized() or tdist.get_world_size() == 1:
        return ms
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


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
    entry = rec.get(workload)
    if not entry or entry.get("kernel_sha256_16") != kernel_source_hash(workload):
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
    """The bf16 tensor peak for a kernel timed over a long loop of calls (seconds
    under the power cap): the sustained figure of MEASURED_PEAKS.json, else the
    pool's earlier sustained measurement, about 1.4 PFLOP/s."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1400.0, "fallback"


def roofline_entry(workload, attn_b, flops, avg_ms, gbs, tflops, hbm_peak, hbm_kind):
    """The attention call's roofline: HBM for decode (about 4 flop/byte at GQA 4),
    the tensor pipe for prefill chunks (a dense contraction)."""
    kern = ("paged_attention call: tcgen05 chunk kernel (S and O accumulated in tensor memory)"
            if workload in ("chunk512_bf16", "chunk512_d256_bf16") else
            "paged_attention call: block-streaming decode kernel + split-K merge kernel, then the "
            "tcgen05 chunk kernel" if workload == "mixed_bf16" else
            "paged_attention call: block-streaming decode kernel + split-K merge kernel")
    common = {"kernel": kern,
              "algorithmic_bytes": attn_b, "algorithmic_flops": flops, "avg_ms": avg_ms,
              "traffic": kernel_traffic(workload)}
    if workload in ("chunk512_bf16", "chunk512_d256_bf16"):
        peak, kind = measured_tensor_peak()
        return dict(common, bound="tensor", achieved=tflops, peak=peak, unit="TFLOP/s",
                    frac=tflops / peak,
                    peak_source="measured (MEASURED_PEAKS.json bf16_tflops_sustained)" if kind == "measured"
                    else "fallback 1.4 PFLOP/s sustained (the calls are timed in a loop of seconds "
                         "under the power cap)")
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


def attention_run_ms(call, stream, n):
    """Device ms per call over n calls issued back to back, between two CUDA
    events on their stream (after 3 untimed calls).  Successive calls overlap
    as they do in a serving loop: a call's kernels are programmatic dependents
    of the previous call's, so its plan runs while the previous call drains."""
    for _ in range(3):
        call()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def sub_batch(batch, idx):
    """Sequences idx of a batch (same pools), with their query rows."""
    qsl = batch["query_start_lens"].tolist()
    toks = torch.cat([torch.arange(qsl[i], qsl[i + 1]) for i in idx])
    lens = torch.tensor([qsl[i + 1] - qsl[i] for i in idx], dtype=torch.int32)
    sub = dict(batch)
    sub["q"] = batch["q"][toks]
    sub["block_tables"] = batch["block_tables"][idx]
    sub["context_lens"] = batch["context_lens"][idx]
    sub["query_start_lens"] = torch.cat([torch.zeros(1, dtype=torch.int32), torch.cumsum(lens, 0)]).to(torch.int32)
    return sub


def mixed_split(batch, pool, device, n_calls, hbm_peak, hbm_kind):
    """A mixed step's decode rows and chunk rows, each as a call of its own
    (same pool, same kernels as in the mixed call): the decode rows against
    the HBM roofline, the chunk rows against the tensor roofline."""
    from paged_kv_cache_chunked_b200 import api
    qn = (batch["query_start_lens"][1:] - batch["query_start_lens"][:-1]).tolist()
    out = {}
    stream = torch.cuda.current_stream(device)
    for name, idx in (("decode_rows", [i for i, n in enumerate(qn) if n == 1]),
                      ("chunk_rows", [i for i, n in enumerate(qn) if n > 1])):
        sb = sub_batch(batch, idx)
        dq, dt_ = sb["q"].to(device), sb["block_tables"].to(device)
        dctx, dqsl = sb["context_lens"].to(device), sb["query_start_lens"].to(device)
        o = torch.empty_like(dq)
        ms = attention_run_ms(lambda: api.paged_attention(
            dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"], out=o), stream, n_calls)
        ab, _, _ = step_bytes(sb)
        fl = attention_flops(sb)
        if name == "decode_rows":
            gbs = ab / (ms * 1e-3) / 1e9
            out[name] = {"sequences": len(idx), "ms": ms, "algorithmic_bytes": ab, "achieved": gbs,
                         "unit": "GB/s", "peak": hbm_peak, "frac": gbs / hbm_peak, "bound": "hbm"}
        else:
            tp, _ = measured_tensor_peak()
            tf = fl / (ms * 1e-3) / 1e12
            out[name] = {"sequences": len(idx), "ms": ms, "algorithmic_flops": fl, "achieved": tf,
                         "unit": "TFLOP/s", "peak": tp, "frac": tf / tp, "bound": "tensor"}
    return out


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
    call = lambda: api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"],
                                       out=out)
    avg = attention_run_ms(call, stream, n_calls)
    iso_each = attention_call_ms(call, stream, n_calls)
    iso = statistics.mean(iso_each)
    assert pool.check_device_errors() == 0
    peak, kind = measured_peak()
    gbs = attn_b / (avg * 1e-3) / 1e9
    r = roofline_entry(name, attn_b, attention_flops(batch), avg, gbs, None, peak, kind)
    r.update(calls=n_calls, isolated_call_ms=iso, isolated_call_median_ms=statistics.median(iso_each),
             config=workload_config(name, batch, f"no flush: {kv_b / 1e6:.0f} MB of KV "
                                                                f"per call, more than the 126 MB L2"))
    del pool
    torch.cuda.empty_cache()
    return r


def indirection_cost(batch, pool, dq, dctx, dqsl, device, n_calls):
    """["Batching and PagedAttention", "The indirection has a cost"]: the same
    decode batch through the same kernel with each sequence's blocks
    contiguous and in logical order (identity tables) against the shuffled
    tables of the workload.  The logical K/V are identical, so the outputs
    must be bit-identical; the ratio of call times is the price of the scatter."""
    from paged_kv_cache_chunked_b200 import api
    tables = batch["block_tables"]
    ctx = batch["context_lens"].tolist()
    bs = batch["block_size"]
    nblk = [-(-c // bs) for c in ctx]
    old_ids = torch.cat([tables[b, :n].long() for b, n in enumerate(nblk)])
    contig = torch.full_like(tables, -1)
    base = 0
    for b, n in enumerate(nblk):
        contig[b, :n] = torch.arange(base, base + n, dtype=torch.int32)
        base += n
    N, Hkv, _, d = batch["k_pool"].shape
    cpool = api.kv_pool_create(N, bs, Hkv, d, torch.bfloat16, device)
    cpool.k_pool[:base] = pool.k_pool[old_ids.to(device)]
    cpool.v_pool[:base] = pool.v_pool[old_ids.to(device)]
    dt_s, dt_c = tables.to(device), contig.to(device)
    o_s, o_c = torch.empty_like(dq), torch.empty_like(dq)
    stream = torch.cuda.current_stream(device)
    call_s = lambda: api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_s, dctx, dqsl, batch["scale"], out=o_s)
    call_c = lambda: api.paged_attention(dq, cpool.k_pool, cpool.v_pool, dt_c, dctx, dqsl, batch["scale"],
                                         out=o_c)
    ms_s, ms_c = [], []
    for _ in range(2):          # alternate, so that both see the same clocks
        ms_s.append(attention_run_ms(call_s, stream, n_calls // 2))
        ms_c.append(attention_run_ms(call_c, stream, n_calls // 2))
    torch.cuda.synchronize(device)
    same = bool(torch.equal(o_s, o_c))
    assert cpool.check_device_errors() == 0
    del cpool
    torch.cuda.empty_cache()
    t_s, t_c = statistics.mean(ms_s), statistics.mean(ms_c)
    return {"shuffled_ms": t_s, "contiguous_ms": t_c, "paged_over_contiguous": t_s / t_c,
            "outputs_bit_identical": same, "calls_each": n_calls // 2 * len(ms_s),
            "pages_figure": "+20-26% for a paged kernel against an optimised contiguous kernel "
                            "(hardware not stated)",
            "how": "one kernel, tables that list each sequence's blocks contiguously in logical order "
                   "against the workload's randomly permuted tables"}


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

    # a step: the new tokens' K/V stored and attention over them, in one call
    # (pk_paged_attention_append; where the block-streaming kernel serves the
    # batch, the attention kernel stores them itself)
    def step():
        api.paged_attention_append(dq, dk, dv, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"],
                                   out=out)

    # the same step as two calls: the append kernel, then attention
    def step_two_calls():
        api.paged_kv_append(dk, dv, dslots, pool=pool)
        api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"], out=out)

    def attention_only():
        api.paged_attention(dq, pool.k_pool, pool.v_pool, dt_, dctx, dqsl, batch["scale"], out=out)

    # the append (unless the decode kernel stores the rows), then per window of
    # 512 sequences: with groups of <= 8 q heads the block-streaming decode
    # kernel and its merge kernel, behind the tcgen05 chunk kernel when chunks
    # are present; else a chunk kernel (when chunks are present) and the
    # tile-streaming decode kernel; the general kernel is one launch
    paths = pool.paths()
    tc = bool(paths & api.PK_PATH_TENSOR_CORE)
    B = batch["context_lens"].shape[0]
    windows = (B + 511) // 512
    blocks = bool(paths & api.PK_PATH_DECODE_BLOCKS) and Hq // Hkv <= 8
    umma = bool(paths & api.PK_PATH_CHUNK_TCGEN05) and 128 % (Hq // Hkv) == 0
    # the block-streaming kernel is followed by its split-K merge kernel
    if blocks and T == B:
        per_window = 2                  # block-streaming decode, merge kernel
    elif blocks and umma:
        per_window = 3                  # tcgen05 chunk kernel, block-streaming decode behind it, merge kernel
    else:
        per_window = 2 if T > B or Hq // Hkv > 16 else 1
    # the new K/V are stored by the block-streaming kernel where it serves a
    # decode-only batch, else by the position append kernel
    stored_in_kernel = blocks and T == B
    launches_per_step = (0 if stored_in_kernel else 1) + (windows * per_window if tc else 1)
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
    # the attention call alone, for its roofline: a separate pass after the
    # timed steps (a step's kernels start as programmatic dependents of the
    # previous ones, and no event sits between them)
    n_attn = max(args.steps, 50)
    attn_avg_ms = attention_run_ms(attention_only, stream, n_attn)
    attn_iso_each = attention_call_ms(attention_only, stream, n_attn)
    attn_iso_ms = statistics.mean(attn_iso_each)
    two_call_ms = attention_run_ms(step_two_calls, stream, n_attn)
    # a long enough window for the clock sampler to see the load
    t_extra = time.perf_counter()
    while not args.profile_run and time.perf_counter() - t_extra < 1.0:
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)
    clk = clocks.stop() if not args.profile_run else {"sm_mhz": None, "reasons": ["not sampled"]}
    assert pool.check_device_errors() == 0

    total_ms = max_over_ranks(total_ms, device)
    ms_per_step = total_ms / args.steps
    value = world * (attn_b + app_b) / (ms_per_step * 1e-3) / 1e9

    # end to end through the public API: every step copies its inputs from
    # pinned host memory and its output back.  Serving overlaps those copies
    # with the kernels, so the timed loop does too: inputs and outputs are
    # double-buffered on the device, host-to-device copies run on one stream
    # and device-to-host copies on another, ordered against the compute stream
    # by events (a step's copy into a buffer waits for the kernels of the step
    # two back that read it).  The same steps with every copy serialised on
    # the compute stream are reported beside it.
    e2e = None
    if not args.no_e2e and not args.profile_run:
        h_in = [x.pin_memory() for x in (batch["q"], k_new, v_new, batch["block_tables"],
                                         batch["context_lens"], batch["query_start_lens"])]
        h_outs = [torch.empty_like(batch["q"]).pin_memory() for _ in range(2)]
        sets = [[torch.empty_like(x, device=device) for x in h_in] for _ in range(2)]
        outs = [torch.empty_like(dq) for _ in range(2)]
        h2d = sum(x.numel() * x.element_size() for x in h_in)
        d2h = h_outs[0].numel() * h_outs[0].element_size()
        h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("h2d", "comp", "d2h")}
        used = [False, False]

        def kernels(bufs, o):
            api.paged_attention_append(bufs[0], bufs[1], bufs[2], pool.k_pool, pool.v_pool, bufs[3], bufs[4],
                                       bufs[5], batch["scale"], out=o)

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(h2d_s):
                if used[j]:
                    h2d_s.wait_event(ev["comp"][j])        # the step two back has read set j
                for dst, src in zip(sets[j], h_in):
                    dst.copy_(src, non_blocking=True)
                ev["h2d"][j].record(h2d_s)
            stream.wait_event(ev["h2d"][j])
            if used[j]:
                stream.wait_event(ev["d2h"][j])           # out[j] of the step two back is home
            kernels(sets[j], outs[j])
            ev["comp"][j].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev["comp"][j])
                h_outs[j].copy_(outs[j], non_blocking=True)
                ev["d2h"][j].record(d2h_s)
            used[j] = True

        def timed(fn):
            s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            if dist:
                tdist.barrier()
            torch.cuda.synchronize(device)
            s2.record(stream)
            h2d_s.wait_event(s2)
            d2h_s.wait_event(s2)
            for i in range(args.steps):
                fn(i)
            for x in (h2d_s, d2h_s):
                done = torch.cuda.Event()
                done.record(x)
                stream.wait_event(done)
            e2.record(stream)
            torch.cuda.synchronize(device)
            e_ms = max_over_ranks(s2.elapsed_time(e2), device)
            return e_ms / args.steps

        def serial_step(i):
            for dst, src in zip(sets[0], h_in):
                dst.copy_(src, non_blocking=True)
            kernels(sets[0], outs[0])
            h_outs[0].copy_(outs[0], non_blocking=True)

        for i in range(4):
            e2e_step(i)
        e_ms = timed(e2e_step)
        ok = bool(torch.equal(h_outs[0], h_outs[1])) and bool(torch.isfinite(h_outs[0].float()).all())
        for i in range(3):
            serial_step(i)
        s_ms = timed(serial_step)
        e2e = {"value": world * (attn_b + app_b) / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "serialized_ms_per_step": s_ms,
               "serialized_value": world * (attn_b + app_b) / (s_ms * 1e-3) / 1e9,
               "how": "per step: host-to-device copies of q, the new K/V, tables, lengths from "
                      "pinned memory; pk_paged_attention_append; device-to-host copy of the output; copies "
                      "overlapped with the neighbouring steps' kernels on two copy streams "
                      "(double-buffered device inputs and outputs); serialized_*: the same with every "
                      "copy on the compute stream"}
        assert ok, "end-to-end outputs differ between the two buffers"

    if rank != 0:
        return
    peak, peak_kind = measured_peak()
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
        "pool_paths": {n: bool(paths & getattr(api, "PK_PATH_" + n))
                       for n in ("TENSOR_CORE", "DECODE_BLOCKS", "CHUNK_TCGEN05")},
        "roofline": roofline_entry(args.workload, attn_b, flops, attn_avg_ms, achieved, tflops,
                                   peak, peak_kind),
        "attention_tflops": tflops,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": dict(clk, window="the timed region plus 1 s of the same steps right after it"),
        "attention_timing": f"{n_attn} attention calls back to back between two CUDA events, in a "
                            f"pass after the timed steps (roofline avg_ms); the same calls each "
                            f"between their own events: isolated_call_ms",
    }
    line["step_call"] = ("pk_paged_attention_append: the new K/V stored "
                         + ("by the block-streaming decode kernel" if stored_in_kernel
                            else "by the position append kernel") + ", then attention")
    line["two_call_ms_per_step"] = two_call_ms
    line["two_call_value"] = world * (attn_b + app_b) / (two_call_ms * 1e-3) / 1e9
    line["two_call"] = "pk_paged_kv_append with slots, then pk_paged_attention, back to back"
    line["roofline"]["isolated_call_ms"] = attn_iso_ms
    line["roofline"]["isolated_call_median_ms"] = statistics.median(attn_iso_each)
    if e2e:
        line["e2e"] = e2e
    if args.workload == "mixed_bf16" and not args.profile_run:
        split = mixed_split(batch, pool, device, max(50, min(args.steps, 500)), peak, peak_kind)
        tp, _ = measured_tensor_peak()
        ideal_ms = (split["decode_rows"]["algorithmic_bytes"] / (peak * 1e9)
                    + split["chunk_rows"]["algorithmic_flops"] / (tp * 1e12)) * 1e3
        line["mixed"] = dict(split, call_ms=attn_avg_ms, ideal_ms=ideal_ms, call_frac=ideal_ms / attn_avg_ms,
                             how="ideal_ms = decode-row bytes / HBM peak + chunk-row flops / bf16 peak; "
                                 "each part also timed alone through the same entry point")
    if args.workload == "decode64_bf16" and not args.profile_run and world == 1:
        clocks2 = ClockSampler(device.index if device.index is not None else 0)
        clocks2.start()
        time.sleep(0.3)
        n_calls = max(50, min(args.steps, 1000))
        line["indirection"] = indirection_cost(batch, pool, dq, dctx, dqsl, device, 2 * n_calls)
        extra = workload_roofline("longdoc_bf16", device, n_calls)
        clk2 = clocks2.stop()
        extra["clocks"] = clk2
        line["indirection"]["clocks"] = clk2
        line["extra_rooflines"] = {"longdoc_bf16": extra}
    if world == 1 and args.cpu_baseline_seconds > 0 and not args.profile_run:
        import oracle
        sec, runs, threads = oracle_step_seconds(batch, args.cpu_baseline_seconds)
        line["cpu_baseline"] = {"value": attn_b / sec / 1e9, "unit": "GB/s", "cores": threads,
                                "kind": "oracle",
                                "sample": f"float64 oracle attention over the whole {args.workload} "
                                          f"batch (attention bytes only), {runs} runs"}
        # the same on one host core, over a leading part of the batch (about a
        # quarter of the budget's worth of all-core runs, at least one sequence)
        B1 = batch["context_lens"].shape[0]
        n1 = max(1, min(B1, int(B1 * min(1.0, args.cpu_baseline_seconds / max(sec * threads, 1e-9)))))
        sub = subset_batch(batch, n1)
        sub_b, _, _ = step_bytes(sub)
        oracle.set_num_threads(1)
        try:
            sec1, runs1, threads1 = oracle_step_seconds(sub, args.cpu_baseline_seconds / 2)
        finally:
            oracle.set_num_threads(threads)
        line["cpu_baseline_1core"] = {"value": sub_b / sec1 / 1e9, "unit": "GB/s", "cores": threads1,
                                      "kind": "oracle",
                                      "sample": f"float64 oracle attention over the first {n1} of {B1} "
                                                f"sequences of {args.workload} on one core, {runs1} runs"}
    print(json.dumps(line), flush=True)


# KV append and block copy alone: the append of a chunked-prefill step of 64
# sequences x 512 tokens (32,768 new tokens) to distinct random slots of a
# decode-64-shaped pool (8 kv heads, head dim 128, 16-token blocks, bf16), then
# 4,096 random whole-block copies (the copy-on-write step of a fork).  The
# append moves 268 MB and the copy 537 MB, both above the 126 MB L2.
KVOPS = dict(num_blocks=9594, n_kv_heads=8, block_size=16, head_dim=128, tokens=32768, pairs=4096,
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
    total_ms = max_over_ranks(start.elapsed_time(end), device)
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
                   "l2": "no flush: the append moves 0.27 GB and the copy 0.54 GB, each more than the 126 MB L2",
                   "parallelism": "replicas"},
        "pct_hbm": 100.0 * value / world / peak,
        "append_gbs": ach, "copy_gbs": copy_b / (copy_ms * 1e-3) / 1e9,
        "roofline": {"kernel": "kv_append (paged_kv_append of 32,768 tokens)", "bound": "hbm",
                     "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                     "algorithmic_bytes": app_b, "avg_ms": app_ms, "traffic": kernel_traffic("append_copy"),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s"},
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


class AttentionSplit:
    """on_step hook of a trace run: after each step's timed region, times the
    step's attention call again, then its decode rows alone (sequences of one
    query token) and its chunk rows alone (several query tokens), each run
    twice back to back between CUDA events on the stream, into scratch outputs
    (the pool is only read).  The second run is the kernel's figure; the first
    follows the host's planning gap, as every serving step does, and is kept
    as the in-loop figure.  A step reads several hundred MB of KV against the
    126 MB L2, so the repeat finds little of it in L2."""

    def __init__(self, runner, record_steps=0):
        self.r = runner
        self.acc = dict(full_ms=0.0, dec_ms=0.0, chunk_ms=0.0, dec_bytes=0, chunk_flops=0, steps=0,
                        dec_calls=0, chunk_calls=0, dec_first_ms=0.0, chunk_first_ms=0.0)
        self.record_steps = record_steps
        self.recorded = []
        self._first = 0.0

    def _time(self, fn):
        st = torch.cuda.current_stream(self.r.device)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(st)
        fn()
        ev[1].record(st)
        fn()
        ev[2].record(st)
        ev[2].synchronize()
        self._first = ev[0].elapsed_time(ev[1])
        return ev[1].elapsed_time(ev[2])

    def __call__(self, plan, t, out):
        from paged_kv_cache_chunked_b200 import api
        if out is None:
            return
        r, dev = self.r, self.r.device
        if len(self.recorded) < self.record_steps:
            self.recorded.append({k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()})
        q = t["q"]
        tables, ctx, qsl = t["tables"], t["ctx"], t["qsl"]
        qn = (qsl[1:] - qsl[:-1]).tolist()
        c = ctx.tolist()
        dtab, dctx, dqsl = tables.to(dev), ctx.to(dev), qsl.to(dev)
        scratch = torch.empty_like(q)
        self.acc["full_ms"] += self._time(lambda: api.paged_attention(
            q, r.pool.k_pool, r.pool.v_pool, dtab, dctx, dqsl, r.scale, out=scratch))
        kv_tok = r.Hkv * r.d * 2 * 2
        dec = [i for i, n in enumerate(qn) if n == 1]
        chk = [i for i, n in enumerate(qn) if n > 1]
        qs = qsl.tolist()
        for idx, is_dec in ((dec, True), (chk, False)):
            if not idx:
                continue
            sel = torch.tensor(idx, dtype=torch.int64)
            toks = torch.cat([torch.arange(qs[i], qs[i + 1]) for i in idx])
            sq = q[toks.to(dev)]
            lens = torch.tensor([qn[i] for i in idx], dtype=torch.int32)
            sqsl = torch.zeros(len(idx) + 1, dtype=torch.int32)
            sqsl[1:] = torch.cumsum(lens, 0)
            stab, sctx = dtab[sel.to(dev)], dctx[sel.to(dev)]
            sqsl = sqsl.to(dev)
            so = torch.empty_like(sq)
            ms = self._time(lambda: api.paged_attention(sq, r.pool.k_pool, r.pool.v_pool, stab, sctx,
                                                        sqsl, r.scale, out=so))
            if is_dec:
                self.acc["dec_ms"] += ms
                self.acc["dec_first_ms"] += self._first
                self.acc["dec_calls"] += 1
                self.acc["dec_bytes"] += (sum(c[i] for i in idx) * kv_tok + 2 * len(idx) * r.Hq * r.d * 2
                                          + sum(-(-c[i] // r.bs) for i in idx) * 4)
            else:
                self.acc["chunk_ms"] += ms
                self.acc["chunk_first_ms"] += self._first
                self.acc["chunk_calls"] += 1
                keys = sum(qn[i] * (c[i] - qn[i]) + qn[i] * (qn[i] + 1) // 2 for i in idx)
                self.acc["chunk_flops"] += 4 * r.Hq * r.d * keys
        self.acc["steps"] += 1

    def summary(self, hbm_peak, tensor_peak):
        a = self.acc
        dec_gbs = a["dec_bytes"] / (a["dec_ms"] * 1e-3) / 1e9 if a["dec_ms"] else None
        ch_tf = a["chunk_flops"] / (a["chunk_ms"] * 1e-3) / 1e12 if a["chunk_ms"] else None
        first_gbs = a["dec_bytes"] / (a["dec_first_ms"] * 1e-3) / 1e9 if a["dec_first_ms"] else None
        return {
            "decode_rows": {"gbs": dec_gbs, "frac_of_hbm_peak": dec_gbs / hbm_peak if dec_gbs else None,
                            "algorithmic_bytes": a["dec_bytes"], "ms": a["dec_ms"], "calls": a["dec_calls"],
                            "gbs_first_call_after_host_gap": first_gbs},
            "chunk_rows": {"tflops": ch_tf, "frac_of_bf16_peak": ch_tf / tensor_peak if ch_tf else None,
                           "flops": a["chunk_flops"], "ms": a["chunk_ms"], "calls": a["chunk_calls"],
                           "ms_first_call_after_host_gap": a["chunk_first_ms"],
                           "share_of_attention_ms": a["chunk_ms"] / a["full_ms"] if a["full_ms"] else None},
            "attention_ms": a["full_ms"], "steps": a["steps"],
            "how": "after each timed step (a second run of the same trace): the step's attention call, "
                   "then its decode rows alone and its chunk rows alone, each twice back to back between "
                   "CUDA events; the second of each pair is the kernel figure"}


def oracle_steps_baseline(recorded, pool_shape, dtype, scale, budget_s, k0=None, v0=None):
    """The oracle as it stands (float64 attention, its append and copy) over the
    recorded steps in order, on a CPU pool, until budget_s seconds are spent."""
    import oracle
    kp = k0.clone() if k0 is not None else torch.zeros(pool_shape, dtype=dtype)
    vp = v0.clone() if v0 is not None else torch.zeros(pool_shape, dtype=dtype)
    done, toks, t0 = 0, 0, time.perf_counter()
    for t in recorded:
        if t["pairs"].shape[0]:
            oracle.block_copy(kp, vp, t["pairs"])
        oracle.kv_append(kp, vp, t["k"], t["v"], t["slots"])
        oracle.paged_attention(t["q"], kp, vp, t["tables"], t["ctx"], t["qsl"], scale)
        done += 1
        toks += t["q"].shape[0]
        if time.perf_counter() - t0 > budget_s:
            break
    sec = time.perf_counter() - t0
    return {"value": toks / sec, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"the first {done} steps in order: oracle block copy, append and float64 "
                      f"attention of every row ({toks} tokens, {sec:.1f} s)"}


def run_serving(args, rank, world, device):
    """Scheduler-driven workloads: the continuous-batching trace (300
    iterations, Poisson arrivals, chunked prefill, preemption) or n-sample
    forks with copy-on-write.  Reports tokens/s per scheduler step over the
    GPU time of copy + append + attention, and KV GB/s."""
    from paged_kv_cache_chunked_b200.drivers import ForkRunner, TraceRunner
    peak, peak_kind = measured_peak()
    tpeak, _ = measured_tensor_peak()
    kv_tok = 8 * 128 * 2 * 2          # K+V bytes per token per layer (8 kv heads, d 128, bf16)
    clocks = ClockSampler(device.index if device.index is not None else 0)
    if not args.profile_run:
        clocks.start()
        time.sleep(0.3)
    extra = {}
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

        def runner():
            return TraceRunner(device, preempt="swap" if swap else "recompute",
                               num_host_blocks=8192 if swap else 0,
                               trace=prefix_trace_requests() if prefix else None,
                               prefix_cache=args.workload == "trace_prefix",
                               num_blocks=6144 if hybrid else 8192, state_slots=64 if hybrid else 0)
        r = runner()
        skip = args.warmup
        wall = 0.0
        while r.sched.step_no < 300 and (r.pending or r.sched.has_work()):
            t0 = time.perf_counter()
            rec = r.step()
            if r.sched.step_no > skip:
                wall += time.perf_counter() - t0
            if rec is not None:
                recs.append(rec)
        recs = [x for x in recs if x.step >= skip]
        cfg = {"workload": args.workload, "steps_run": r.sched.step_no, "warmup_steps": skip,
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
        plan_s = sum(x.host_plan_ms for x in recs) / 1e3
        values_s = sum(x.host_values_ms for x in recs) / 1e3
        values_gpu_s = sum(x.values_gpu_ms or 0.0 for x in recs) / 1e3
        extra["wall_clock"] = {
            "tokens_per_s": sum(toks) / wall, "s": wall, "steps": len(recs),
            "host_planning_s": plan_s, "value_generation_launch_s": values_s,
            "value_generation_gpu_s": values_gpu_s,
            "tokens_per_s_without_value_generation_gpu_time": sum(toks) / (wall - values_gpu_s),
            "how": "host time of the timed scheduler steps, each ending in a wait for its kernels: "
                   "planning (schedule + complete, host_planning_s), launching the generation of the "
                   "step's synthetic q/k/v on the GPU (a stand-in for the model; its kernels run "
                   "before the step's timed region), host-to-device copies of the step's metadata, "
                   "the step's kernels and the wait"}
        if not args.profile_run:
            del r
            torch.cuda.empty_cache()
            # the same trace with the host one step ahead: step n + 1 is planned
            # and launched while step n runs (TraceRunner.step(wait=False))
            r3 = runner()
            toks3, t3 = 0, None
            while r3.sched.step_no < 300 and (r3.pending or r3.sched.has_work()):
                if t3 is None and r3.sched.step_no >= skip:
                    r3.finish()
                    torch.cuda.synchronize(device)
                    t3 = time.perf_counter()
                rec3 = r3.step(wait=False)
                if rec3 is not None and rec3.step >= skip:
                    toks3 += rec3.tokens
            r3.finish()
            torch.cuda.synchronize(device)
            wall3 = time.perf_counter() - t3
            extra["wall_clock"].update(
                overlapped_tokens_per_s=toks3 / wall3, overlapped_s=wall3,
                overlapped_how="a third run of the same trace: the host plans and launches step n + 1 "
                               "while step n runs (at most one step in flight), timed from the first "
                               "timed step to the end of the last one's kernels")
            del r3
            torch.cuda.empty_cache()
            r2 = runner()
            split = AttentionSplit(r2, record_steps=30 if world == 1 and args.workload == "trace" else 0)
            while r2.sched.step_no < 300 and (r2.pending or r2.sched.has_work()):
                r2.step(on_step=split)
            extra["attention_split"] = split.summary(peak, tpeak)
            if split.recorded and args.cpu_baseline_seconds > 0:
                shape = tuple(r2.pool.k_pool.shape)
                del r2
                torch.cuda.empty_cache()
                extra["cpu_baseline"] = oracle_steps_baseline(split.recorded, shape, torch.bfloat16,
                                                              128 ** -0.5, 2 * args.cpu_baseline_seconds)
    else:
        plen = 1028 if args.workload == "fork1028" else 1024

        def fork_run(bs, n_steps, record=0):
            r = ForkRunner(device, prompt_len=plen, block_size=bs)
            r.prefill()
            for _ in range(min(args.warmup, 8)):
                r.decode_step()
            ms, toks, kvb, copies, rec = [], [], [], 0, []
            steps = min(n_steps, r.decode_steps - min(args.warmup, 8))
            for _ in range(steps):
                before_unique = r.unique_blocks()
                t, c = r.decode_step()
                ms.append(t)
                toks.append(len(r.seqs))
                kvb.append(before_unique * bs * kv_tok)     # unique (physical) blocks read
                copies += c
            st = r.bm.stats()
            info = {"block_size": bs, "tokens_per_s": sum(toks) / (sum(ms) * 1e-3),
                    "kv_gbs_unique": sum(kvb) / (sum(ms) * 1e-3) / 1e9, "decode_steps_timed": steps,
                    "unique_blocks": r.unique_blocks(), "clone_blocks": r.clone_blocks(),
                    "tail_waste_slots": st["tail_waste_slots"], "copies": copies}
            del r
            torch.cuda.empty_cache()
            return ms, toks, kvb, copies, info

        ms, toks, kvb, copies, info = fork_run(16, args.steps)
        cfg = {"workload": args.workload, "prompts": 64, "prompt_len": plen, "samples": 4,
               "block_size": 16, "n_q_heads": 32, "n_kv_heads": 8, "head_dim": 128,
               "decode_steps_timed": info["decode_steps_timed"], "unique_blocks": info["unique_blocks"],
               "clone_blocks": info["clone_blocks"], "copies": copies}
        useful = sum(toks)
        if not args.profile_run:
            # "Choosing the block size": the same fork workload at blocks of 8, 16 and 32
            extra["block_size_sweep"] = {str(b): (info if b == 16 else fork_run(b, args.steps)[4])
                                         for b in (8, 16, 32)}
            if world == 1 and args.cpu_baseline_seconds > 0:
                # the oracle over the first 8 decode steps after the prefill
                rb = ForkRunner(device, prompt_len=plen, block_size=16, decode_steps=8)
                rb.prefill()
                torch.cuda.synchronize()
                k0, v0 = rb.pool.k_pool.cpu(), rb.pool.v_pool.cpu()
                rec = []
                for _ in range(8):
                    rb.decode_step(on_step=lambda t, out: rec.append(
                        {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()}), timed=False)
                shape = tuple(rb.pool.k_pool.shape)
                del rb
                torch.cuda.empty_cache()
                extra["cpu_baseline"] = oracle_steps_baseline(rec, shape, torch.bfloat16, 128 ** -0.5,
                                                              2 * args.cpu_baseline_seconds, k0, v0)
    clk = clocks.stop() if not args.profile_run else {"sm_mhz": None, "reasons": ["not sampled"]}
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
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6.65 TB/s",
            "timing": "per-step CUDA events around swaps + copy + append and attention (trace: one "
                      "pk_paged_attention_append call; fork: append, then attention); host scheduling "
                      "excluded (see wall_clock)",
            "clocks": dict(clk, window="the whole run: timed steps and the measurement passes after them"),
            **extra}
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
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
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
    clk = clocks.stop()
    base = study["continuous_4096"]
    line = {"metric": METRIC, "value": base["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
            "steps": base["steps"], "warmup": 0, "ms_per_step": base["gpu_ms"] / base["steps"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "policy", "trace": "trace_requests(arrivals 1.0/step, 300 steps, seed 1004)",
                       "requests": len(trace), "num_blocks": 8192, "block_size": 16, "max_chunk": 512},
            "study": study,
            "clocks": dict(clk, window="every configuration of the study"),
            "timing": "per-step CUDA events around the block copy and the append + attention call, summed; "
                      "host scheduling excluded"}
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
