"""Iteration-level scheduler on the host (no GPU).

* The same trace planned with the C++ block manager and with the oracle block
  manager yields identical steps: requests, slots, copy pairs and block
  tables bit for bit.
* Invariants from the pages: the token cap holds every step, decodes come
  before prefill chunks, chunks are at most 512 tokens, preemption evicts the
  latest arrival with all of its blocks, every finished request produced its
  output length, every block returns to the pool at the end.
"""

import torch

from oracle import OracleBlockManager
from paged_kv_cache_chunked_b200.api import BlockManager
from paged_kv_cache_chunked_b200.scheduler import Request, Scheduler
from paged_kv_cache_chunked_b200.workloads import trace_requests


class OracleAdapter:
    """The oracle block manager behind the interface the scheduler uses."""

    def __init__(self, num_blocks, block_size):
        self.o = OracleBlockManager(num_blocks, block_size)
        self.num_blocks, self.block_size = num_blocks, block_size

    def __getattr__(self, name):
        return getattr(self.o, name)

    def fill_tables(self, seqs, width):
        out = torch.full((len(seqs), width), -1, dtype=torch.int32)
        for i, s in enumerate(seqs):
            t = self.o.block_table(s)
            out[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
        return out

    def stats(self):
        return self.o.stats()

    def refcount(self, block):
        return self.o.refcount[block]


def _run(bm, trace, n_steps, budget=4096, chunk=512, preempt="recompute"):
    sched = Scheduler(bm, token_budget=budget, max_chunk=chunk, preempt=preempt)
    pending = [Request(i, a, p, o) for i, (a, p, o) in enumerate(trace)]
    plans = []
    step = 0
    while step < n_steps or sched.has_work():
        while pending and pending[0].arrival <= step:
            sched.add_request(pending.pop(0))
        plan = sched.schedule()
        plans.append(plan)
        _check_plan(plan, sched, budget, chunk)
        sched.complete(plan)
        step += 1
        if step > 20 * n_steps:
            raise AssertionError("trace did not drain")
    return sched, plans


def _check_plan(plan, sched, budget, chunk):
    assert plan.num_tokens <= budget
    seen = set()
    phase_decode = True
    for req, n, start in zip(plan.requests, plan.counts, plan.starts):
        assert req.rid not in seen
        seen.add(req.rid)
        is_decode = start >= req.target
        if is_decode:
            assert phase_decode, "a decode after a prefill chunk"
            assert n == 1
        else:
            phase_decode = False
            assert 1 <= n <= chunk and start + n <= req.target
    assert len(plan.slots) == plan.num_tokens
    assert len(set(plan.slots)) == len(plan.slots)


def _small_trace():
    # a shortened, denser version of the serving trace: a small pool so that
    # preemption and recomputation happen
    return trace_requests(n_steps=40, arrivals_per_step=3.0, prompt_median=300, prompt_max=2000,
                          out_min=5, out_max=60, seed=77)


def test_product_and_oracle_managers_plan_identically():
    trace = _small_trace()
    s1, p1 = _run(BlockManager(600, 16), trace, 40)
    s2, p2 = _run(OracleAdapter(600, 16), trace, 40)
    assert len(p1) == len(p2)
    for a, b in zip(p1, p2):
        assert [r.rid for r in a.requests] == [r.rid for r in b.requests]
        assert a.counts == b.counts and a.starts == b.starts
        assert a.slots == b.slots and a.copy_pairs == b.copy_pairs
        assert torch.equal(a.tables, b.tables)
    assert s1.metrics == s2.metrics
    assert s1.metrics["preemptions"] > 0      # the small pool forces preemption


def test_trace_invariants_and_drain():
    trace = _small_trace()
    bm = BlockManager(600, 16)
    sched, plans = _run(bm, trace, 40)
    assert len(sched.finished) == len(trace)
    for r in sched.finished:
        assert r.generated == r.output_len
        assert len(r.token_steps) == r.output_len
        assert r.stored == r.prompt_len + r.output_len - 1
        assert r.first_token_step >= r.arrival
    assert bm.num_free() == 600 and bm.stats()["num_seqs"] == 0


def test_preemption_picks_latest_arrival_and_frees_all_blocks():
    bm = BlockManager(6, 4)                 # 24 slots
    sched = Scheduler(bm, token_budget=64, max_chunk=64)
    a, b = Request(0, 0, 12, 10), Request(1, 1, 12, 10)
    sched.add_request(a)
    sched.add_request(b)
    sched.complete(sched.schedule())        # both prefilled: 3 + 3 full blocks, pool full
    assert bm.num_free() == 0 and a.generated == 1 and b.generated == 1
    plan = sched.schedule()                  # a's decode needs a block: b is evicted
    assert [r.rid for r in plan.preempted] == [1]
    assert b.seq == -1 and b.stored == 0 and b.target == 12
    assert [r.rid for r in plan.requests] == [0]
    sched.complete(plan)
    assert bm.num_free() == 2               # b's three blocks came back, a took one


def test_request_larger_than_pool_is_rejected_early():
    sched = Scheduler(BlockManager(4, 4), token_budget=64, max_chunk=64)
    try:
        sched.add_request(Request(0, 0, 15, 5))
    except ValueError as e:
        assert "more than the pool" in str(e)
    else:
        raise AssertionError("not rejected")


# ---------------------------------------------------------------- swap mode
def _swap_run(bm, host_blocks=400):
    bm.set_host_blocks(host_blocks)
    return _run(bm, _small_trace(), 40, preempt="swap")


def test_swap_mode_product_and_oracle_managers_plan_identically():
    s1, p1 = _swap_run(BlockManager(600, 16))
    s2, p2 = _swap_run(OracleAdapter(600, 16))
    assert len(p1) == len(p2)
    for a, b in zip(p1, p2):
        assert [r.rid for r in a.requests] == [r.rid for r in b.requests]
        assert a.counts == b.counts and a.starts == b.starts
        assert a.slots == b.slots and a.copy_pairs == b.copy_pairs
        assert a.swap_ops == b.swap_ops
        assert torch.equal(a.tables, b.tables)
    assert s1.metrics == s2.metrics
    assert s1.metrics["swaps_out"] > 0 and s1.metrics["swaps_in"] == s1.metrics["swaps_out"]


def test_swap_mode_resumes_without_recomputation_and_drains():
    # a swapped request keeps its tokens: every request stores exactly
    # prompt + output - 1 positions, each written once, with no recompute
    # prefill; every device and host block is back at the end
    trace = _small_trace()
    bm = BlockManager(600, 16)
    sched, plans = _swap_run(bm)
    assert len(sched.finished) == len(trace)
    written = {}
    for plan in plans:
        for req, s, n in zip(plan.requests, plan.starts, plan.counts):
            for pos in range(s, s + n):
                assert (req.rid, pos) not in written, "a position written twice"
                written[(req.rid, pos)] = plan.step
    for r in sched.finished:
        assert r.generated == r.output_len and r.stored == r.prompt_len + r.output_len - 1
        assert sum(1 for (rid, _) in written if rid == r.rid) == r.stored
    assert sched.metrics["preemptions"] == sched.metrics["swaps_out"] > 0
    st = bm.stats()
    assert st["free_blocks"] == 600 and st["host_free_blocks"] == 400 and st["num_seqs"] == 0


def test_swap_ins_bring_back_exactly_what_was_swapped_out():
    # all blocks of a sequence move together: every swap-in returns the very
    # host blocks one earlier swap-out filled, and each op names distinct blocks
    bm = BlockManager(600, 16)
    sched, plans = _swap_run(bm)
    on_host = []
    for plan in plans:
        for to_host, pairs in plan.swap_ops:
            src = [a for a, _ in pairs]
            dst = [b for _, b in pairs]
            assert len(set(src)) == len(src) and len(set(dst)) == len(dst)
            if to_host:
                on_host.append(frozenset(dst))
            else:
                assert frozenset(src) in on_host
                on_host.remove(frozenset(src))
    assert on_host == []


def test_small_host_pool_falls_back_to_recompute():
    # victims the host pool cannot hold are recomputed, as in recompute mode
    bm = BlockManager(600, 16)
    bm.set_host_blocks(8)
    sched, _ = _run(bm, _small_trace(), 40, preempt="swap")
    assert len(sched.finished) == len(_small_trace())
    assert sched.metrics["preemptions"] > sched.metrics["swaps_out"]


# ---------------------------------------------------------------- prefix cache
def _prefix_trace():
    from paged_kv_cache_chunked_b200.workloads import prefix_trace_requests
    return prefix_trace_requests(n_steps=40, arrivals_per_step=3.0, sys_lens=(200, 64, 320),
                                 user_median=100, user_max=800, out_min=5, out_max=60, seed=78)


def _prefix_run(bm, prefix_cache=True, n_steps=40):
    sched = Scheduler(bm, token_budget=4096, max_chunk=512, prefix_cache=prefix_cache)
    pending = [Request(i, a, p, o, group=g, sys_len=sl) for i, (a, p, o, g, sl) in enumerate(_prefix_trace())]
    plans = []
    step = 0
    while step < n_steps or sched.has_work():
        while pending and pending[0].arrival <= step:
            sched.add_request(pending.pop(0))
        plan = sched.schedule()
        plans.append(plan)
        _check_plan(plan, sched, 4096, 512)
        sched.complete(plan)
        step += 1
        assert step < 20 * n_steps, "trace did not drain"
    return sched, plans


def test_prefix_cache_product_and_oracle_managers_plan_identically():
    s1, p1 = _prefix_run(BlockManager(600, 16))
    s2, p2 = _prefix_run(OracleAdapter(600, 16))
    assert len(p1) == len(p2)
    for a, b in zip(p1, p2):
        assert [r.rid for r in a.requests] == [r.rid for r in b.requests]
        assert a.starts == b.starts and a.counts == b.counts and a.slots == b.slots
        assert torch.equal(a.tables, b.tables)
    assert s1.metrics == s2.metrics and s1.metrics["prefix_hit_tokens"] > 0


def test_prefix_cache_skips_exactly_the_shared_tokens_and_drains():
    # each request's shared-prompt blocks come from the cache when another
    # request wrote them; every other position is written exactly once, and
    # every block (cached ones included) is back in the pool at the end
    bm = BlockManager(600, 16)
    sched, plans = _prefix_run(bm)
    cold, _ = _prefix_run(BlockManager(600, 16), prefix_cache=False)
    written = {}
    for plan in plans:
        for req, s, n in zip(plan.requests, plan.starts, plan.counts):
            for pos in range(s, s + n):
                written[(req.rid, pos)] = written.get((req.rid, pos), 0) + 1
    hit = sched.metrics["prefix_hit_tokens"]
    assert hit > 0 and len(sched.finished) == len(_prefix_trace())
    for r in sched.finished:
        mine = [pos for (rid, pos) in written if rid == r.rid]
        skipped = r.stored - len(mine)
        assert skipped % 16 == 0 and skipped <= r.sys_len        # whole shared blocks only
        assert all(pos >= skipped for pos in mine)               # the skipped part is the prefix
    if sched.metrics["preemptions"] == 0 and cold.metrics["preemptions"] == 0:
        tokens = lambda s: sum(r.stored for r in s.finished)
        assert sum(written.values()) == tokens(sched) - hit
    st = bm.stats()
    assert st["free_blocks"] == 600 and st["cached_blocks"] == 0 and st["prefix_hits"] * 16 == hit


# ---------------------------------------------------------------- static batching
from paged_kv_cache_chunked_b200.scheduler import StaticScheduler  # noqa: E402


def _run_policy(sched, reqs, limit=5000):
    pending = sorted(reqs, key=lambda r: (r.arrival, r.rid))
    step = 0
    plans = []
    while pending or sched.has_work():
        while pending and pending[0].arrival <= step:
            sched.add_request(pending.pop(0))
        plan = sched.schedule()
        plans.append((plan, set(getattr(sched, "batch", set()))))
        sched.complete(plan)
        step += 1
        assert step < limit, "did not drain"
    return plans


def test_static_batching_runs_each_batch_to_its_end():
    # "a batch that runs until every member has finished, then the next batch
    # starts" [Batching and PagedAttention, "Static batching"]
    reqs = [Request(i, a, p, o) for i, (a, p, o) in enumerate(_small_trace())]
    sched = StaticScheduler(BlockManager(600, 16), batch_size=8, token_budget=4096, max_chunk=512)
    plans = _run_policy(sched, reqs)
    batches = []
    for plan, batch in plans:
        assert len(batch) <= 8
        assert {r.rid for r in plan.requests} <= batch
        if batch and (not batches or batch - batches[-1]):
            batches.append(set(batch))
    for a, b in zip(batches, batches[1:]):
        assert not (a & b)                              # a new batch only after the old one ended
    assert len(sched.finished) == len(reqs) and sched.batches == len(batches)


def _toy(lengths, prompt=16):
    return [Request(i, 0, prompt, o) for i, o in enumerate(lengths)]


def test_continuous_batching_finishes_mixed_lengths_sooner():
    # [Batching and PagedAttention, "Try it" 1]: 4 slots, mixed output lengths;
    # the average request finishes sooner with continuous batching
    lengths = [10, 500, 30, 200, 20, 300, 50, 100, 10, 400, 60, 15]
    cont = Scheduler(BlockManager(4096, 16), token_budget=4096, max_chunk=512, max_seqs=4)
    stat = StaticScheduler(BlockManager(4096, 16), batch_size=4, token_budget=4096, max_chunk=512)
    _run_policy(cont, _toy(lengths))
    _run_policy(stat, _toy(lengths))
    mean = lambda s: sum(r.finish_step for r in s.finished) / len(s.finished)
    assert mean(cont) < 0.8 * mean(stat)
    assert max(r.finish_step for r in cont.finished) <= max(r.finish_step for r in stat.finished)


def test_equal_lengths_make_static_and_continuous_batching_alike():
    # [Batching and PagedAttention, "Try it" 2]: with similar lengths continuous
    # batching barely helps; with equal ones every request finishes at the same
    # step under both policies
    lengths = [40] * 12
    cont = Scheduler(BlockManager(4096, 16), token_budget=4096, max_chunk=512, max_seqs=4)
    stat = StaticScheduler(BlockManager(4096, 16), batch_size=4, token_budget=4096, max_chunk=512)
    _run_policy(cont, _toy(lengths))
    _run_policy(stat, _toy(lengths))
    fin = lambda s: sorted((r.rid, r.finish_step) for r in s.finished)
    assert fin(cont) == fin(stat)


def test_summary_converts_steps_to_gpu_time():
    # a request arriving at step 0 with tokens at steps 2, 3 and 5, steps of
    # 1..6 ms: first token at the end of step 2 (1+2+3 = 6 ms), gaps of 4 ms
    # (step 3) and 5 + 6 = 11 ms (steps 4 and 5)
    from paged_kv_cache_chunked_b200.scheduler import summary
    r = Request(0, 0, 100, 3)
    r.admit_step, r.first_token_step, r.token_steps = 0, 2, [2, 3, 5]
    out = summary([r], step_ms=[1.0, 2.0, 3.0, 4.0, 5.0, 6.0])["all"]
    assert out["ttft_ms"]["mean"] == 6.0
    assert out["itl_ms"]["mean"] == 7.5 and out["ttft"]["mean"] == 2 and out["itl"]["mean"] == 1.5


# ---------------------------------------------------------------- two pools
def test_two_pool_admission_caps_concurrency_at_the_state_slots():
    # [7.8 PagedAttention & continuous batching, "01 Concept"]: with a
    # fixed-size state slot per sequence beside the KV blocks, no more
    # requests run than there are slots; both managers plan identically
    def run(bm):
        bm.set_state_slots(6)
        sched, plans = _run(bm, _small_trace(), 40)
        return sched, plans
    s1, p1 = run(BlockManager(600, 16))
    s2, p2 = run(OracleAdapter(600, 16))
    assert [[r.rid for r in a.requests] for a in p1] == [[r.rid for r in b.requests] for b in p2]
    assert max(len(p.requests) for p in p1) == 6
    assert len(s1.finished) == len(_small_trace())
    assert s1.bm.stats()["state_free_slots"] == 6


# ---------------------------------------------------------------- property test
from hypothesis import given, settings, HealthCheck, strategies as hst  # noqa: E402


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(
    reqs=hst.lists(hst.tuples(hst.integers(0, 12), hst.integers(1, 300), hst.integers(1, 40),
                              hst.integers(-1, 2), hst.integers(0, 160)), min_size=1, max_size=25),
    nb=hst.integers(40, 200), bs=hst.sampled_from([4, 16]), budget=hst.sampled_from([64, 256, 1024]),
    mode=hst.sampled_from(["recompute", "swap"]), prefix=hst.booleans(), static=hst.sampled_from([None, 3]))
def test_random_traces_plan_identically_and_drain(reqs, nb, bs, budget, mode, prefix, static):
    # any small trace, pool, budget and mode: the C++ and oracle managers give
    # the same plans, every plan keeps the invariants, and everything drains
    reqs = sorted(reqs)
    trace = []
    for a, p, o, g, sl in reqs:
        if -(-(p + o - 1) // bs) > nb:
            continue                                    # would be rejected at admission
        trace.append((a, p, o, g, min(sl, p - 1) if g >= 0 else 0))
    if not trace:
        return

    def run(bm):
        if mode == "swap":
            bm.set_host_blocks(nb)
        kw = dict(token_budget=budget, max_chunk=min(budget, 128), preempt=mode, prefix_cache=prefix)
        sched = StaticScheduler(bm, static, **kw) if static else Scheduler(bm, **kw)
        pending = [Request(i, a, p, o, group=g, sys_len=sl) for i, (a, p, o, g, sl) in enumerate(trace)]
        plans, step = [], 0
        while pending or sched.has_work():
            while pending and pending[0].arrival <= step:
                sched.add_request(pending.pop(0))
            plan = sched.schedule()
            _check_plan(plan, sched, budget, min(budget, 128))
            plans.append(([r.rid for r in plan.requests], plan.starts, plan.counts, plan.slots,
                          plan.copy_pairs, plan.swap_ops, plan.tables.tolist()))
            sched.complete(plan)
            step += 1
            assert step < 5000, "did not drain"
        return sched, plans

    s1, p1 = run(BlockManager(nb, bs))
    s2, p2 = run(OracleAdapter(nb, bs))
    assert p1 == p2 and s1.metrics == s2.metrics
    assert len(s1.finished) == len(trace)
    st = s1.bm.stats()
    assert st["free_blocks"] == nb and st["num_seqs"] == 0 and st["cached_blocks"] == 0


def test_step_value_keys_match_the_per_request_keys():
    # The serving driver builds a step's generator keys with array operations.
    # They must equal, row by row in batch order, the per-request keys: a
    # request's own id past its shared system prompt, the prompt's id inside it.
    from paged_kv_cache_chunked_b200.drivers import TraceRunner
    from paged_kv_cache_chunked_b200.workloads import SYS_VID_BASE, prefix_trace_requests
    trace = prefix_trace_requests()[:60]
    sched = Scheduler(BlockManager(2048, 16), token_budget=1024, max_chunk=256, prefix_cache=True)
    pending = [Request(i, *t[:3], group=t[3], sys_len=t[4]) for i, t in enumerate(trace)]
    step = checked = shared = 0
    while (pending or sched.has_work()) and step < 400:
        while pending and pending[0].arrival <= step:
            sched.add_request(pending.pop(0))
        plan = sched.schedule()
        if plan.requests:
            vid, pos = TraceRunner.value_keys(plan)
            want_v, want_p = [], []
            for req, s, n in zip(plan.requests, plan.starts, plan.counts):
                want_v += TraceRunner.value_ids(req, s, n)
                want_p += list(range(s, s + n))
            assert vid.tolist() == want_v and pos.tolist() == want_p
            checked += 1
            shared += int((vid >= SYS_VID_BASE).sum())
        sched.complete(plan)
        step += 1
    assert checked > 20 and shared > 0


def test_step_values_in_one_pass_equal_the_per_stream_values():
    # the drivers draw a step's q, k and v with one hash pass over the keys;
    # each must be bit for bit the per-stream generator's output
    from paged_kv_cache_chunked_b200.workloads import SYS_VID_BASE, token_values, token_values_qkv
    g = torch.Generator().manual_seed(5)
    rids = torch.randint(0, 400, (257,), generator=g)
    rids[::7] = SYS_VID_BASE + 3
    pos = torch.randint(0, 9000, (257,), generator=g)
    q, k, v = token_values_qkv(1004, rids, pos, 32, 8, 128, torch.bfloat16)
    for stream, (got, heads) in enumerate(((q, 32), (k, 8), (v, 8))):
        want = token_values(1004, stream, rids, pos, heads, 128, torch.bfloat16)
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
