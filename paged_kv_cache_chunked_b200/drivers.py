"""Drivers that run the paged-KV calls the way a serving engine does.

TraceRunner   continuous batching over an arrival trace: each iteration the
              scheduler plans a mixed batch (decodes first, then prefill
              chunks), the kernels run swaps -> copy -> append + attention
              (one call) on one stream, finished requests are freed ["PagedAttention &
              Continuous Batching" (study notes), "Continuous batching" and
              "Flow"; "Batching and PagedAttention", "Continuous batching"].
              Preempted requests are recomputed, or with preempt="swap" their
              blocks go to a pinned host pool and back ["Batching and
              PagedAttention", "When blocks run out"].  With prefix_cache and
              a trace of shared system prompts, a request starts on the
              blocks of its system prompt that another request already wrote
              ["Batching and PagedAttention", "Sharing blocks"].
ForkRunner    n parallel samples of each prompt: prefill, fork (children share
              the prompt's blocks by reference count), then decode steps in
              which the first write into a shared, partly filled tail block
              triggers copy-on-write [study notes, "Copy-on-write";
              "Batching and PagedAttention", "Sharing blocks"].

Both generate queries and K/V with the counter-based generator of
`workloads.token_values`, keyed by (request id, position), on the device.
"""

import time

import numpy as np
import torch

from . import api
from .scheduler import Request, Scheduler, StaticScheduler
from .workloads import SYS_VID_BASE, token_values_qkv, trace_requests


class StepRecord:
    """One scheduler step: its batch, its GPU time (CUDA events around swaps,
    copies, append and attention) and its host time split into planning
    (schedule + complete), launching the generation of the step's synthetic
    q/k/v (which stands in for the model; values_gpu_ms is its GPU time) and the
    rest (metadata copies, launches, the wait)."""
    __slots__ = ("step", "tokens", "decode_rows", "prefill_tokens", "copies", "gpu_ms",
                 "context_tokens", "num_seqs", "swap_blocks", "new_tokens", "host_plan_ms",
                 "host_values_ms", "values_gpu_ms", "host_total_ms")

    def __init__(self, **kw):
        for k, v in kw.items():
            setattr(self, k, v)


class TraceRunner:
    """Runs the serving trace through the scheduler and the GPU kernels."""

    def __init__(self, device, num_blocks=8192, block_size=16, n_q_heads=32, n_kv_heads=8,
                 head_dim=128, token_budget=4096, max_chunk=512, trace=None, seed=1004,
                 n_steps=300, dtype=torch.bfloat16, preempt="recompute", num_host_blocks=0,
                 prefix_cache=False, max_seqs=None, static_batch=None, state_slots=0):
        self.device = torch.device(device)
        self.Hq, self.Hkv, self.d, self.bs = n_q_heads, n_kv_heads, head_dim, block_size
        self.dtype = dtype
        self.seed = seed
        self.n_steps = n_steps
        self.pool = api.kv_pool_create(num_blocks, block_size, n_kv_heads, head_dim, dtype,
                                       self.device)
        self.bm = api.BlockManager(num_blocks, block_size)
        if state_slots:          # two pools: a fixed-size state slot per sequence beside the KV blocks
            self.bm.set_state_slots(state_slots)
        self.host = None
        if preempt == "swap":
            self.bm.set_host_blocks(num_host_blocks)
            self.host = api.host_pool_create(num_host_blocks, self.pool)
        kw = dict(token_budget=token_budget, max_chunk=max_chunk, preempt=preempt,
                  prefix_cache=prefix_cache, max_seqs=max_seqs)
        self.sched = (StaticScheduler(self.bm, static_batch, **kw) if static_batch
                      else Scheduler(self.bm, **kw))
        trace = trace if trace is not None else trace_requests(n_steps=n_steps, seed=seed)
        # (arrival, prompt, output) or (arrival, prompt, output, group, system prompt length)
        self.pending = [Request(i, *t[:3], group=t[3], sys_len=t[4]) if len(t) == 5 else Request(i, *t)
                        for i, t in enumerate(trace)]
        self.scale = head_dim ** -0.5
        self.records = []
        self.rejected = 0
        self.high_water = {}     # request id -> positions stored at least once
        self._inflight = []      # (record, events) of steps whose GPU time is not read yet

    def _admit_arrivals(self, step):
        while self.pending and self.pending[0].arrival <= step:
            req = self.pending.pop(0)
            try:
                self.sched.add_request(req)
            except ValueError:
                self.rejected += 1

    def step(self, on_step=None, timed=True, wait=True):
        """One iteration.  on_step(plan, tensors, out) is called after the
        kernels (for parity checks).  Returns the step's record, or None when
        there was nothing to run.

        wait=False (no on_step): the step returns once its kernels are
        launched, and its GPU time is read at the next step or in finish().
        The host then plans and launches step n + 1 while step n runs, as a
        serving loop does; the scheduler's state never depends on a step's
        results, only on its plan.  At most one step is left in flight."""
        t_start = time.perf_counter()
        step = self.sched.step_no
        self._admit_arrivals(step)
        plan = self.sched.schedule()
        t_planned = time.perf_counter()
        dev = self.device
        swaps = [(to_host, torch.tensor(pairs, dtype=torch.int32).reshape(-1, 2).pin_memory().to(
                     dev, non_blocking=True)) for to_host, pairs in plan.swap_ops]
        if not plan.requests:
            # nothing to run but, possibly, swaps decided while planning (timed:
            # they are part of the serving work)
            rec = None
            if swaps:
                stream = torch.cuda.current_stream(dev)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                self._run_swaps(swaps)
                e1.record(stream)
                if on_step is not None:
                    on_step(plan, {"swaps": plan.swap_ops}, None)
                e1.synchronize()
                rec = StepRecord(step=step, tokens=0, decode_rows=0, prefill_tokens=0, copies=0,
                                 gpu_ms=e0.elapsed_time(e1), context_tokens=0, num_seqs=0,
                                 swap_blocks=sum(len(p) for _, p in plan.swap_ops), new_tokens=0,
                                 host_values_ms=0.0, values_gpu_ms=0.0)
                self.records.append(rec)
            t_c = time.perf_counter()
            self.sched.complete(plan)
            if rec is not None:
                t_end = time.perf_counter()
                rec.host_plan_ms = 1e3 * ((t_planned - t_start) + (t_end - t_c))
                rec.host_total_ms = 1e3 * (t_end - t_start)
            return rec
        rids, pos = self.value_keys(plan)
        meta = {
            "tables": plan.tables,
            "ctx": torch.tensor(plan.context_lens, dtype=torch.int32),
            "qsl": torch.tensor(plan.query_start_lens(), dtype=torch.int32),
            "pairs": torch.tensor(plan.copy_pairs, dtype=torch.int32).reshape(-1, 2),
        }
        # the fused call stores each row at position c_b - q_b + i through the
        # block tables, so the slots are not sent; a step hook gets them
        # staged through pinned memory: a copy from pageable memory would first
        # wait for the stream, and with it for the step still running
        d = {k: v.pin_memory().to(dev, non_blocking=True) for k, v in meta.items()}
        if on_step is not None:
            meta["slots"] = torch.tensor(plan.slots, dtype=torch.int64)
        stream = torch.cuda.current_stream(dev)
        t_v = time.perf_counter()
        if timed:
            ev_v = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev_v[0].record(stream)
        q, k, v = token_values_qkv(self.seed, rids, pos, self.Hq, self.Hkv, self.d, self.dtype, dev)
        if timed:
            ev_v[1].record(stream)
        t_v = time.perf_counter() - t_v
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        self._run_swaps(swaps)
        if d["pairs"].shape[0]:
            api.block_copy(d["pairs"], pool=self.pool)
        out = api.paged_attention_append(q, k, v, self.pool.k_pool, self.pool.v_pool, d["tables"], d["ctx"],
                                         d["qsl"], self.scale)
        if timed:
            e1.record(stream)
        if on_step is not None:
            on_step(plan, {"q": q, "k": k, "v": v, "swaps": plan.swap_ops, **meta}, out)
        n_dec = sum(1 for r, s in zip(plan.requests, plan.starts) if s >= r.target)
        # positions written for the first time (a recompute prefill rewrites
        # positions a preempted request had already stored)
        new = 0
        for req, s, n in zip(plan.requests, plan.starts, plan.counts):
            hw = self.high_water.get(req.rid, 0)
            new += max(0, s + n - max(s, hw))
            self.high_water[req.rid] = max(hw, s + n)
        rec = StepRecord(step=step, tokens=plan.num_tokens, decode_rows=n_dec,
                         prefill_tokens=plan.num_tokens - n_dec, copies=len(plan.copy_pairs),
                         gpu_ms=None, context_tokens=sum(plan.context_lens), num_seqs=len(plan.requests),
                         swap_blocks=sum(len(p) for _, p in plan.swap_ops), new_tokens=new,
                         host_values_ms=1e3 * t_v, values_gpu_ms=None)
        if timed:
            self._inflight.append((rec, e0, e1, ev_v))
            self._settle(0 if wait or on_step is not None else 1)
        t_c = time.perf_counter()
        self.sched.complete(plan)
        t_end = time.perf_counter()
        rec.host_plan_ms = 1e3 * ((t_planned - t_start) + (t_end - t_c))
        rec.host_total_ms = 1e3 * (t_end - t_start)
        self.records.append(rec)
        return rec

    @staticmethod
    def value_ids(req, start, n):
        """Generator key of positions start .. start+n-1 of req: its system
        prompt's for the shared prefix, its own after it."""
        if req.group < 0:
            return [req.rid] * n
        shared = SYS_VID_BASE + req.group
        return [shared if p < req.sys_len else req.rid for p in range(start, start + n)]

    @staticmethod
    def value_keys(plan):
        """Generator keys of the step's rows, in batch order: (value id,
        position) per row, value_ids of every request concatenated, built with
        array operations (a chunked step has thousands of rows)."""
        counts = np.asarray(plan.counts, dtype=np.int64)
        first = np.repeat(np.cumsum(counts) - counts, counts)
        pos = np.repeat(np.asarray(plan.starts, dtype=np.int64), counts) + (np.arange(int(counts.sum())) - first)
        reqs = plan.requests
        rid = np.repeat(np.asarray([r.rid for r in reqs], dtype=np.int64), counts)
        grp = np.repeat(np.asarray([r.group for r in reqs], dtype=np.int64), counts)
        sys_len = np.repeat(np.asarray([r.sys_len for r in reqs], dtype=np.int64), counts)
        vid = np.where((grp >= 0) & (pos < sys_len), SYS_VID_BASE + grp, rid)
        return torch.from_numpy(vid), torch.from_numpy(pos)

    def _run_swaps(self, swaps):
        # in the order the scheduler decided them: a swap-in may reuse blocks a
        # swap-out of the same step freed, and the reverse on the host
        for to_host, pairs in swaps:
            if pairs.shape[0]:
                api.swap_blocks(pairs, to_host=to_host, host_pool=self.host, pool=self.pool)

    def step_ms(self):
        """GPU ms of every scheduler step so far (0 for steps with no work)."""
        ms = [0.0] * self.sched.step_no
        for r in self.records:
            ms[r.step] = r.gpu_ms or 0.0
        return ms

    def _settle(self, keep):
        """Read the GPU times of all but the last `keep` steps in flight (each
        waits for its step's kernels)."""
        while len(self._inflight) > keep:
            rec, e0, e1, ev_v = self._inflight.pop(0)
            e1.synchronize()
            rec.gpu_ms = e0.elapsed_time(e1)
            rec.values_gpu_ms = ev_v[0].elapsed_time(ev_v[1])

    def finish(self):
        """Wait for the steps in flight and fill in their GPU times."""
        self._settle(0)

    def run(self, max_steps=None, on_step=None, wait=True):
        limit = max_steps if max_steps is not None else self.n_steps
        while self.sched.step_no < limit and (self.pending or self.sched.has_work()):
            self.step(on_step, wait=wait)
        self.finish()
        return self.records


class ForkRunner:
    """n parallel samples per prompt sharing the prompt's blocks (copy-on-write)."""

    def __init__(self, device, n_prompts=64, prompt_len=1024, n_samples=4, block_size=16,
                 n_q_heads=32, n_kv_heads=8, head_dim=128, decode_steps=256, seed=1005,
                 dtype=torch.bfloat16, chunk=512, fused=False):
        self.device = torch.device(device)
        # fused: a decode step's append and attention as one call (the copy-on-
        # write copies first; the rows then go through the updated tables)
        self.fused = fused
        self.Hq, self.Hkv, self.d, self.bs = n_q_heads, n_kv_heads, head_dim, block_size
        self.dtype, self.seed, self.chunk = dtype, seed, chunk
        self.n_prompts, self.prompt_len, self.n_samples = n_prompts, prompt_len, n_samples
        self.decode_steps = decode_steps
        per_seq = -(-(prompt_len + decode_steps) // block_size)
        # shared prompt blocks + a private copy of the rest for every sample, with slack
        self.num_blocks = n_prompts * n_samples * per_seq + 64
        self.pool = api.kv_pool_create(self.num_blocks, block_size, n_kv_heads, head_dim, dtype,
                                       self.device)
        self.bm = api.BlockManager(self.num_blocks, block_size)
        self.scale = head_dim ** -0.5
        self.seqs = []       # (seq id, key id for the generator)
        self.lengths = []
        self.total_copies = 0

    def _values(self, keys, pos):
        dev = self.device
        q, k, v = token_values_qkv(self.seed, keys, pos, self.Hq, self.Hkv, self.d, self.dtype, dev)
        return q, k, v

    def prefill(self):
        """Prefill every prompt in chunks (causal), then fork n-1 children each."""
        parents = [self.bm.add_seq() for _ in range(self.n_prompts)]
        done = 0
        while done < self.prompt_len:
            n = min(self.chunk, self.prompt_len - done)
            keys, pos, slots = [], [], []
            for i, s in enumerate(parents):
                sl, pairs = self.bm.append_slots(s, n)
                assert not pairs
                slots.extend(sl)
                keys.extend([i * self.n_samples] * n)     # the parent's key: sample 0
                pos.extend(range(done, done + n))
            q, k, v = self._values(keys, pos)
            dev = self.device
            api.paged_kv_append(k, v, torch.tensor(slots, dtype=torch.int64, device=dev), pool=self.pool)
            width = -(-(done + n) // self.bs)
            tables = self.bm.fill_tables(parents, width).to(dev)
            ctx = torch.full((len(parents),), done + n, dtype=torch.int32, device=dev)
            qsl = torch.arange(0, (len(parents) + 1) * n, n, dtype=torch.int32, device=dev)
            api.paged_attention(q, self.pool.k_pool, self.pool.v_pool, tables, ctx, qsl, self.scale)
            done += n
        for i, p in enumerate(parents):
            self.seqs.append((p, i * self.n_samples))
            for j in range(1, self.n_samples):
                self.seqs.append((self.bm.fork(p), i * self.n_samples + j))
        self.lengths = [self.prompt_len] * len(self.seqs)

    def decode_step(self, on_step=None, timed=True):
        """One decode token for every sample: copy-on-write pairs, append, attend.
        Samples of one prompt diverge: each has its own key for new tokens."""
        slots, pairs, keys, pos = [], [], [], []
        for (s, key), L in zip(self.seqs, self.lengths):
            sl, pr = self.bm.append_slots(s, 1)
            slots.extend(sl)
            pairs.extend(pr)
            keys.append(key)
            pos.append(L)
        self.lengths = [L + 1 for L in self.lengths]
        dev = self.device
        q, k, v = self._values(keys, pos)
        width = -(-max(self.lengths) // self.bs)
        tables = self.bm.fill_tables([s for s, _ in self.seqs], width)
        meta = {"slots": torch.tensor(slots, dtype=torch.int64), "tables": tables,
                "ctx": torch.tensor(self.lengths, dtype=torch.int32),
                "qsl": torch.arange(len(self.seqs) + 1, dtype=torch.int32),
                "pairs": torch.tensor(pairs, dtype=torch.int32).reshape(-1, 2)}
        dd = {kk: vv.to(dev, non_blocking=True) for kk, vv in meta.items()}
        stream = torch.cuda.current_stream(dev)
        if timed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        if dd["pairs"].shape[0]:
            api.block_copy(dd["pairs"], pool=self.pool)
        if self.fused:
            out = api.paged_attention_append(q, k, v, self.pool.k_pool, self.pool.v_pool, dd["tables"],
                                             dd["ctx"], dd["qsl"], self.scale)
        else:
            api.paged_kv_append(k, v, dd["slots"], pool=self.pool)
            out = api.paged_attention(q, self.pool.k_pool, self.pool.v_pool, dd["tables"], dd["ctx"],
                                      dd["qsl"], self.scale)
        if timed:
            e1.record(stream)
        if on_step is not None:
            on_step({"q": q, "k": k, "v": v, **meta}, out)
        self.total_copies += len(pairs)
        if timed:
            e1.synchronize()
            return e0.elapsed_time(e1), len(pairs)
        return None, len(pairs)

    def unique_blocks(self):
        return self.bm.num_used()

    def clone_blocks(self):
        """Blocks the same samples would hold if every fork cloned its prefix."""
        return sum(-(-L // self.bs) for L in self.lengths)
