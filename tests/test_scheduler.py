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


def _run(bm, trace, n_steps, budget=4096, chunk=512):
    sched = Scheduler(bm, token_budget=budget, max_chunk=chunk)
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
