"""Iteration-level scheduler (continuous batching) driving the paged KV calls.

What the pages fix:
  * every iteration admits new work (a full prefill or one chunk of it),
    drops finished requests and frees their blocks, and runs one mixed batch
    of whatever remains ["PagedAttention & Continuous Batching" (study notes),
    "Continuous batching"; "Batching and PagedAttention", "Continuous
    batching"; "7.8 PagedAttention & continuous batching", "01 Concept"];
  * long prompts are split into chunks so one prefill does not stall every
    decode ["Batching and PagedAttention", "Continuous batching"];
  * a cap on the tokens processed per step bounds the prefill work any step
    absorbs ["Batching and PagedAttention", "Scheduling is a policy"];
    admission reasons in blocks [deep dive, "01 Concept"];
  * first come, first served; when blocks run out, the most recently arrived
    requests are preempted first, all of their blocks together, and later
    recomputed from the tokens they had ["Batching and PagedAttention",
    "When blocks run out"].

Readings where the pages give no number or order (listed in the design notes):
  * token budget 4096 per step, prefill chunks of at most 512 tokens;
  * decodes are scheduled first, one token each, in arrival order; then
    prefill chunks, first come first served, while the budget lasts and the
    chunk's blocks are free (no preemption to admit a prefill);
  * a decode that cannot get a block preempts the latest-arrived running
    request (possibly itself) until it fits;
  * a preempted request goes back to the waiting queue in arrival order; its
    recompute prefill covers its prompt and every generated token but the
    last, which the next decode step appends;
  * a request's K/V and queries are a deterministic function of (request id,
    position), so recomputation reproduces the same bits.

Swap mode (preempt="swap") takes the pages' other option for a victim: its
blocks move to CPU memory, all together, and come back before it runs again
["Batching and PagedAttention", "When blocks run out"].  Readings:
  * the victim keeps its state (tokens stored, generated); a victim that
    shares a block, or that the host pool cannot hold, is recomputed instead;
  * swapped requests come back first, in arrival order, as soon as their
    blocks and one more fit (just their blocks when nothing runs), never in
    the step that swapped them out; while any request is swapped out no new
    request is admitted;
  * the swaps of a step run, in the order they were decided, before its
    copy-on-write copies, appends and attention (a swap-in may land in blocks
    a swap-out of the same step just freed).

Prefix cache (prefix_cache=True): a request whose prompt starts with a shared
system prompt starts on the cached blocks of that prompt, when another request
already wrote them, and prefills only the rest ["Batching and PagedAttention",
"Sharing blocks": requests that share a system prompt can share its blocks,
the basis of prefix caching].  Readings:
  * a block is named by (system prompt, block index), which names its whole
    token prefix; only blocks wholly inside the system prompt are cached, and
    at least one prompt token is always prefilled (its query yields the first
    output token);
  * admission reasons in the blocks the first chunk needs after the hit;
  * a request's system-prompt blocks enter the cache once the step that
    filled them has run.

Two pools: when the block manager also keeps a fixed-size state slot per
sequence (hybrid models), admission needs a free slot as well as the first
chunk's blocks; a recomputed request gives its slot back, a swapped one keeps
it ["7.8 PagedAttention & continuous batching", "01 Concept": two pools with
different lifecycles].

A request with prompt length P and output length O stores P + O - 1 tokens:
the last prefill chunk yields the first output token, each decode step
appends the previous output token and yields the next.
"""

import bisect
from dataclasses import dataclass, field

import torch


@dataclass(eq=False)         # a request is itself: identity, not field-wise, equality
class Request:
    rid: int
    arrival: int
    prompt_len: int
    output_len: int
    seq: int = -1            # block manager sequence, -1 when holding no blocks
    stored: int = 0          # positions whose K/V is in the pool
    target: int = 0          # positions to prefill before decoding
    generated: int = 0       # output tokens produced
    first_token_step: int = -1
    admit_step: int = -1
    finish_step: int = -1
    preemptions: int = 0
    swapped_step: int = -1
    group: int = -1          # shared system prompt, -1 for none
    sys_len: int = 0         # tokens of the shared system prompt at the start of the prompt
    token_steps: list = field(default_factory=list)

    def __post_init__(self):
        self.target = self.prompt_len

    @property
    def prefilling(self):
        return self.stored < self.target


@dataclass
class StepPlan:
    """One iteration's batch: per scheduled request, `n` new positions starting
    at `start`, with the slots, copy-on-write pairs, swaps and block tables the
    step's kernels need (the drivers turn them into device tensors)."""
    step: int
    requests: list          # Request objects, batch order
    starts: list            # first new position per request
    counts: list            # new positions per request
    slots: list             # slot id of every new position, batch order
    copy_pairs: list        # (src, dst) copy-on-write pairs to run first
    context_lens: list      # tokens stored per request after this step's append
    tables: torch.Tensor    # int32 [B, W] block tables (host)
    preempted: list         # requests preempted while planning this step
    swap_ops: list = field(default_factory=list)  # (to_host, [(src, dst), ...]) in order

    @property
    def num_tokens(self):
        return sum(self.counts)

    def query_start_lens(self):
        q = [0]
        for n in self.counts:
            q.append(q[-1] + n)
        return q


def _arrival_order(r):
    return (r.arrival, r.rid)


class Scheduler:
    def __init__(self, bm, token_budget=4096, max_chunk=512, preempt="recompute", prefix_cache=False,
                 max_seqs=None):
        if preempt not in ("recompute", "swap"):
            raise ValueError("preempt must be 'recompute' or 'swap'")
        self.bm = bm
        self.block_size = bm.block_size
        self.token_budget = token_budget
        self.max_chunk = max_chunk
        self.preempt_mode = preempt
        self.prefix_cache = prefix_cache
        self.max_seqs = max_seqs     # cap on requests holding blocks at once ("slots"); None: memory only
        # two pools: the manager's state-slot pool, if it has one (set before the scheduler is made)
        self._state_pool = bool(bm.stats().get("state_slots", 0))
        self.waiting = []    # arrival order
        self.running = []    # arrival order; hold blocks
        self.swapped = []    # arrival order; blocks in the host pool
        self.finished = []
        self.step_no = 0
        self._swap_ops = []  # swaps decided since the last plan was handed out
        self.metrics = {"preemptions": 0, "alloc_failures": 0, "admitted": 0, "swaps_out": 0,
                        "swaps_in": 0, "prefix_hit_tokens": 0}

    def add_request(self, req):
        """Queue a request; one that could never fit in the whole pool is
        rejected here, with the reason, instead of failing mid-generation."""
        total = req.prompt_len + req.output_len - 1
        if -(-total // self.block_size) > self.bm.num_blocks:
            self.metrics["rejected"] = self.metrics.get("rejected", 0) + 1
            raise ValueError(f"request {req.rid} needs {total} tokens, more than the pool holds")
        self._requeue(req)

    def _requeue(self, req):
        bisect.insort(self.waiting, req, key=_arrival_order)

    def has_work(self):
        return bool(self.waiting or self.running or self.swapped)

    # -- preemption -------------------------------------------------------
    def _can_swap_out(self, req):
        table = self.bm.block_table(req.seq)
        return (self.bm.stats()["host_free_blocks"] >= len(table)
                and all(self.bm.refcount(b) == 1 for b in table))

    def _preempt(self, req):
        if self.preempt_mode == "swap" and self._can_swap_out(req):
            self._swap_ops.append((True, self.bm.swap_out(req.seq)))
            req.preemptions += 1
            req.swapped_step = self.step_no
            self.metrics["preemptions"] += 1
            self.metrics["swaps_out"] += 1
            self.running.remove(req)
            bisect.insort(self.swapped, req, key=_arrival_order)
            return
        self.bm.free(req.seq)
        req.seq = -1
        req.stored = 0
        req.target = req.prompt_len + max(req.generated - 1, 0)
        req.preemptions += 1
        self.metrics["preemptions"] += 1
        self.running.remove(req)
        self._requeue(req)

    def _may_admit(self, req):
        """Continuous batching: any waiting request may join at any step."""
        return True

    def _prefix_keys(self, req):
        """Cache keys of the request's blocks that lie wholly inside its system
        prompt, leaving at least one prompt token to prefill."""
        if not self.prefix_cache or req.group < 0:
            return []
        n = min(req.sys_len, req.prompt_len - 1) // self.block_size
        return [((req.group + 1) << 32) | i for i in range(n)]

    def _latest_running(self):
        return max(self.running, key=lambda r: (r.arrival, r.rid))

    # -- one iteration ------------------------------------------------------
    def schedule(self):
        """Plan the next step: reserve slots, emit copy pairs and tables.  If
        requests hold blocks but none can advance (every one of them is
        mid-prefill and the pool is full), the latest arrival is preempted
        and the step planned again."""
        plan = self._plan()
        while not plan.requests and self.running:
            victim = self._latest_running()
            self._preempt(victim)
            plan = self._plan()
            plan.preempted.append(victim)
        plan.swap_ops, self._swap_ops = self._swap_ops, []
        return plan

    def _swap_in_ready(self):
        """Bring swapped requests back, in arrival order, while they fit."""
        for req in list(self.swapped):
            if req.swapped_step == self.step_no:
                break
            need = len(self.bm.block_table(req.seq)) + (1 if self.running else 0)
            if need > self.bm.num_free():
                break        # arrival order: later ones wait behind this one
            self._swap_ops.append((False, self.bm.swap_in(req.seq)))
            self.swapped.remove(req)
            bisect.insort(self.running, req, key=_arrival_order)
            self.metrics["swaps_in"] += 1

    def _plan(self):
        if self.swapped:
            self._swap_in_ready()
        budget = self.token_budget
        batch, starts, counts, slots, pairs, preempted = [], [], [], [], [], []

        def reserve(req, n):
            s, p = self.bm.append_slots(req.seq, n)
            batch.append(req)
            starts.append(req.stored)
            counts.append(n)
            slots.extend(s)
            pairs.extend(p)

        # decodes first, in arrival order: one manager call serves them until one
        # needs a block while none is free; that one preempts the latest arrival
        # (never a request already served: they all arrived earlier) until it
        # fits or is itself preempted, and the rest follow
        decodes = [r for r in self.running if not r.prefilling]     # running is kept in arrival order
        i = 0
        while i < len(decodes) and budget > 0:
            todo = decodes[i:i + budget]
            done, got_slots, got_pairs = self.bm.append_one_each([r.seq for r in todo])
            served = todo[:done]
            batch.extend(served)
            starts.extend([r.stored for r in served])
            counts.extend([1] * done)
            slots.extend(got_slots)
            pairs.extend(got_pairs)
            budget -= done
            i += done
            if done < len(todo):
                req = todo[done]
                while req in self.running and self.bm.blocks_needed(req.seq, 1) > self.bm.num_free():
                    victim = self._latest_running()
                    self.metrics["alloc_failures"] += 1
                    self._preempt(victim)
                    preempted.append(victim)
                decodes = decodes[:i] + [r for r in decodes[i:] if r in self.running]
        # prefill chunks: running requests mid-prefill, then waiting ones (FCFS);
        # nothing new is admitted while a request is swapped out
        in_batch = set(batch)
        candidates = [r for r in self.running if r.prefilling and r not in in_batch]
        if not self.swapped:
            candidates += list(self.waiting)     # filtered below, as they come
        for req in candidates:
            if budget == 0:
                break
            if req.seq < 0 and (req in preempted or not self._may_admit(req)):
                continue
            if req.seq < 0:
                if self.max_seqs is not None and len(self.running) >= self.max_seqs:
                    break        # every slot is taken
                if self._state_pool and self.bm.stats()["state_free_slots"] == 0:
                    break        # two pools: no free per-sequence state slot
                # admission: reason in blocks before taking any (after the
                # prefix-cache hit, whose blocks are already in the pool)
                keys = self._prefix_keys(req)
                hits = self.bm.cached_prefix(keys) if keys else 0
                start = hits * self.block_size
                n = min(self.max_chunk, req.target - start, budget)
                need = -(-(start + n) // self.block_size) - hits
                if need > self.bm.num_free():
                    break        # FCFS: later arrivals wait behind this one
                if keys:
                    req.seq, hits = self.bm.add_seq_cached(keys)
                    req.stored = hits * self.block_size
                    self.metrics["prefix_hit_tokens"] += req.stored
                else:
                    req.seq = self.bm.add_seq()
                if req.admit_step < 0:
                    req.admit_step = self.step_no
                self.waiting.remove(req)
                bisect.insort(self.running, req, key=_arrival_order)
                self.metrics["admitted"] += 1
            n = min(self.max_chunk, req.target - req.stored, budget)
            if self.bm.blocks_needed(req.seq, n) > self.bm.num_free():
                break
            reserve(req, n)
            budget -= n

        seqs = [r.seq for r in batch]
        ctx = [s + n for s, n in zip(starts, counts)]
        width = max([-(-c // self.block_size) for c in ctx] + [1])
        tables = self.bm.fill_tables(seqs, width) if seqs else torch.empty((0, 1), dtype=torch.int32)
        return StepPlan(self.step_no, batch, starts, counts, slots, pairs, ctx, tables, preempted)

    def complete(self, plan):
        """Advance request state after the step's kernels ran; free finished."""
        for req, n in zip(plan.requests, plan.counts):
            was_prefill = req.stored < req.target
            req.stored += n
            if was_prefill and self.prefix_cache and req.group >= 0:
                keys = self._prefix_keys(req)
                full = min(len(keys), req.stored // self.block_size)
                if full:
                    self.bm.cache_blocks(req.seq, keys[:full])
            if was_prefill:
                if req.stored == req.target and req.generated == 0:
                    req.generated = 1
                    req.first_token_step = plan.step
                    req.token_steps.append(plan.step)
            else:
                req.generated += 1
                req.token_steps.append(plan.step)
            if req.generated >= req.output_len and not req.prefilling:
                req.finish_step = plan.step
                self.bm.free(req.seq)
                req.seq = -1
                self.running.remove(req)
                self.finished.append(req)
        self.step_no += 1

    def step_metrics(self):
        s = self.bm.stats()
        return {"free_blocks": s["free_blocks"], "used_blocks": s["used_blocks"],
                "tail_waste_slots": s["tail_waste_slots"], "running": len(self.running),
                "waiting": len(self.waiting), "swapped": len(self.swapped),
                "preemptions": self.metrics["preemptions"],
                "alloc_failures": self.metrics["alloc_failures"]}


class StaticScheduler(Scheduler):
    """Static batching, the comparison the pages draw ["Batching and
    PagedAttention", "Static batching": requests are grouped into a batch that
    runs until every member has finished, then the next batch starts; slots
    of finished members sit idle, new arrivals wait for the whole batch].

    Only admission differs from Scheduler: when no request runs and no batch
    is open, the next batch_size waiting requests (arrival order) become the
    batch; only its members are admitted (their prefill chunks still follow
    the token cap), and the batch closes when all of them have finished.
    Preempted members stay members."""

    def __init__(self, bm, batch_size, **kw):
        super().__init__(bm, **kw)
        self.batch_size = batch_size
        self.batch = set()       # request ids of the open batch
        self.batches = 0

    def _plan(self):
        if not self.batch and not self.running and not self.swapped and self.waiting:
            self.batch = {r.rid for r in self.waiting[:self.batch_size]}
            self.batches += 1
        return super()._plan()

    def _may_admit(self, req):
        return req.rid in self.batch

    def complete(self, plan):
        super().complete(plan)
        self.batch -= {r.rid for r in plan.requests if r.finish_step == plan.step}


def summary(finished, step_ms=None):
    """Per-request serving metrics over finished requests, in scheduler steps
    [7.8 PagedAttention & continuous batching, "01 Concept": queue delay, time
    to first token, inter-token latency], split by request class (prompt
    shorter or longer than 512 tokens) so throughput does not hide starvation.
    With step_ms (GPU ms of each step), time to first token and inter-token
    latency are also given in ms of GPU time: a request arriving at step a
    whose first token comes at step f waits from the start of a to the end of
    f."""
    def stats(xs):
        if not xs:
            return None
        xs = sorted(xs)
        return {"mean": sum(xs) / len(xs), "p50": xs[len(xs) // 2], "p90": xs[int(0.9 * (len(xs) - 1))],
                "max": xs[-1]}

    out = {}
    for name, sel in (("all", lambda r: True), ("short_prompt", lambda r: r.prompt_len <= 512),
                      ("long_prompt", lambda r: r.prompt_len > 512)):
        rs = [r for r in finished if sel(r)]
        itl = []
        for r in rs:
            itl += [b - a for a, b in zip(r.token_steps, r.token_steps[1:])]
        out[name] = {"requests": len(rs),
                     "queue_delay": stats([r.admit_step - r.arrival for r in rs]),
                     "ttft": stats([r.first_token_step - r.arrival for r in rs]),
                     "itl": stats(itl),
                     "preempted": sum(1 for r in rs if r.preemptions)}
        if step_ms is not None:
            end = [0.0]
            for m in step_ms:
                end.append(end[-1] + m)          # end[s + 1]: GPU ms at the end of step s
            at = lambda s: end[min(s, len(end) - 1)]
            itl_ms = []
            for r in rs:
                itl_ms += [at(b + 1) - at(a + 1) for a, b in zip(r.token_steps, r.token_steps[1:])]
            out[name]["ttft_ms"] = stats([at(r.first_token_step + 1) - at(r.arrival) for r in rs])
            out[name]["itl_ms"] = stats(itl_ms)
    return out


def plan_inputs(plan, seed, n_q_heads, n_kv_heads, head_dim, dtype, device):
    """q, k, v for a plan's new positions from the counter-based generator."""
    from .workloads import token_values
    rids, pos = [], []
    for req, s, n in zip(plan.requests, plan.starts, plan.counts):
        rids.extend([req.rid] * n)
        pos.extend(range(s, s + n))
    q = token_values(seed, 0, rids, pos, n_q_heads, head_dim, dtype, device)
    k = token_values(seed, 1, rids, pos, n_kv_heads, head_dim, dtype, device)
    v = token_values(seed, 2, rids, pos, n_kv_heads, head_dim, dtype, device)
    return q, k, v
