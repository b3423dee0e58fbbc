"""The serving drivers on the GPU, step by step against the oracle.

TraceRunner: continuous batching with chunked prefill, preemption and
recomputation; every step's decode rows and a sample of its prefill rows are
compared with the float64 oracle run on a CPU mirror of the pool that the
oracle's own append and copy keep up to date; the GPU pool itself is compared
with the mirror bit for bit.

ForkRunner: parallel samples share their prompt's blocks until a write
["PagedAttention & Continuous Batching" (study notes), "Copy-on-write"]:
siblings read identical K/V before the first decode, the first write into a
shared, partly filled tail copies it (one copy per sharer but the last), and
attention matches the oracle every step.
"""

import pytest
import torch

import oracle
from paged_kv_cache_chunked_b200.drivers import ForkRunner, TraceRunner
from paged_kv_cache_chunked_b200.workloads import trace_requests

from helpers import assert_close

pytestmark = pytest.mark.gpu


class Mirror:
    """CPU copy of the pool (and of the host pool, when swapping) kept current
    with the oracle's swaps, append and copy."""

    def __init__(self, pool, host=None):
        self.k = pool.k_pool.cpu()
        self.v = pool.v_pool.cpu()
        if host is not None:
            self.hk, self.hv = host.k.clone(), host.v.clone()

    def swaps(self, ops):
        for to_host, pairs in ops:     # in the order the scheduler decided them
            if pairs:
                oracle.swap_blocks(self.k, self.v, self.hk, self.hv, pairs, to_host)

    def apply(self, pairs, k, v, slots):
        if pairs.shape[0]:
            oracle.block_copy(self.k, self.v, pairs)
        oracle.kv_append(self.k, self.v, k.cpu(), v.cpu(), slots)


def _check_rows(mirror, t, out, rows, scale, what):
    ref = oracle.paged_attention_rows(t["q"].cpu(), mirror.k, mirror.v, t["tables"], t["ctx"],
                                      t["qsl"], scale, rows)
    got = torch.stack([out[r, h].cpu() for r, h in rows])
    assert_close(got, ref, torch.bfloat16, what)


def _check_tokens(mirror, t, out, toks, n_heads, scale, what):
    """Every q head of the listed query tokens against the oracle."""
    if not toks:
        return
    rows = [(tk, h) for tk in toks for h in range(n_heads)]
    ref = oracle.paged_attention_rows(t["q"].cpu(), mirror.k, mirror.v, t["tables"], t["ctx"],
                                      t["qsl"], scale, rows)
    got = out[torch.tensor(toks, device=out.device)].cpu().reshape(len(rows), -1)
    assert_close(got, ref, torch.bfloat16, what)


def _checked_trace_step(runner, mirror, gen, full_every=None, mirror_every=10):
    """on_step callback: the oracle's append and copy keep the CPU mirror of the
    pool current; every decode row is checked with all its q heads; chunk rows
    are the first, last and a random token (one random head each) of every
    chunk, or, on every full_every-th step, every row of the batch; every
    mirror_every-th step the GPU pool equals the mirror bit for bit."""
    def on_step(plan, t, out):
        mirror.swaps(t["swaps"])
        if out is None:
            return
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        qsl = t["qsl"].tolist()
        what = f"step {plan.step}"
        if full_every and (plan.step + 1) % full_every == 0:
            ref = oracle.paged_attention(t["q"].cpu(), mirror.k, mirror.v, t["tables"], t["ctx"],
                                         t["qsl"], runner.scale)
            assert_close(out, ref, torch.bfloat16, what + ": every row")
        else:
            dec, rows = [], []
            for i, (req, s) in enumerate(zip(plan.requests, plan.starts)):
                toks = list(range(qsl[i], qsl[i + 1]))
                if s >= req.target:
                    dec.append(toks[0])
                else:
                    pick = {toks[0], toks[-1], toks[int(torch.randint(len(toks), (1,), generator=gen))]}
                    rows += [(tk, int(torch.randint(runner.Hq, (1,), generator=gen))) for tk in pick]
            _check_tokens(mirror, t, out, dec, runner.Hq, runner.scale, what + ": decode rows")
            if rows:
                _check_rows(mirror, t, out, rows, runner.scale, what + ": chunk rows")
        if (plan.step + 1) % mirror_every == 0:
            torch.cuda.synchronize()
            assert torch.equal(runner.pool.k_pool.cpu(), mirror.k), what
            assert torch.equal(runner.pool.v_pool.cpu(), mirror.v), what
    return on_step


def test_trace_at_the_stated_geometry(cuda_dev):
    # The continuous-batching trace at its stated size ["Batching and
    # PagedAttention", "Continuous batching": every step admits work, runs one
    # mixed batch of decodes and prefill chunks, long prompts split into chunks]:
    # 8,192-block pool, 32 q / 8 kv heads, head dim 128, block 16, Poisson(4)
    # arrivals, lognormal prompts (median 512, clipped at 8,192) in 512-token
    # chunks, outputs 10..500, budget 4,096 tokens a step.  Steps 1..30: every
    # decode row on every step, every row of the batch on steps 10, 20 and 30,
    # and the GPU pool against the oracle's mirror bit for bit on those steps.
    runner = TraceRunner(cuda_dev)
    assert (runner.bm.num_blocks, runner.Hq, runner.Hkv, runner.d, runner.bs) == (8192, 32, 8, 128, 16)
    assert (runner.sched.token_budget, runner.sched.max_chunk) == (4096, 512)
    mirror = Mirror(runner.pool)
    runner.run(max_steps=30, on_step=_checked_trace_step(runner, mirror, torch.Generator().manual_seed(4),
                                                         full_every=10))
    recs = runner.records
    assert runner.sched.step_no == 30 and len(recs) >= 28    # a step without arrivals has no record
    assert {9, 19, 29} <= {r.step for r in recs}             # the every-row steps ran
    assert sum(r.decode_rows for r in recs) > 0 and sum(r.prefill_tokens for r in recs) > 0
    assert any(r.decode_rows and r.prefill_tokens for r in recs)      # mixed steps were checked
    assert runner.pool.check_device_errors() == 0


def test_static_batching_trace_matches_the_oracle(cuda_dev):
    # static batching ["Batching and PagedAttention", "Static batching"]: a
    # batch is admitted as a whole and runs until its last member finishes;
    # the kernels see the same calls as under continuous batching
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=5, out_max=40, seed=18)
    runner = TraceRunner(cuda_dev, num_blocks=600, n_steps=30, trace=trace, token_budget=1024,
                         max_chunk=256, static_batch=8)
    mirror = Mirror(runner.pool)
    runner.run(max_steps=60, on_step=_checked_trace_step(runner, mirror, torch.Generator().manual_seed(5)))
    assert len(runner.sched.finished) > 0
    assert runner.pool.check_device_errors() == 0


@pytest.mark.parametrize("token_budget", [512, 2048])
def test_token_budget_trace_matches_the_oracle(cuda_dev, token_budget):
    # a smaller and a larger per-step token cap ["Batching and PagedAttention",
    # "Scheduling is a policy"]: the batches change, the kernels' results do not
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=5, out_max=40, seed=19)
    runner = TraceRunner(cuda_dev, num_blocks=400, n_steps=30, trace=trace, token_budget=token_budget,
                         max_chunk=256)
    mirror = Mirror(runner.pool)
    runner.run(max_steps=40, on_step=_checked_trace_step(runner, mirror, torch.Generator().manual_seed(6)))
    assert max(r.tokens for r in runner.records) <= token_budget
    assert runner.pool.check_device_errors() == 0


def test_two_pool_trace_matches_the_oracle(cuda_dev):
    # a fixed-size state slot per sequence beside the paged KV ["7.8
    # PagedAttention & continuous batching", "01 Concept": two pools with
    # different lifecycles]: admission needs a slot too, so at most 6 requests
    # run at once; attention over the KV pool is unchanged
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=5, out_max=40, seed=20)
    runner = TraceRunner(cuda_dev, num_blocks=400, n_steps=30, trace=trace, token_budget=1024,
                         max_chunk=256, state_slots=6)
    mirror = Mirror(runner.pool)
    slots_seen = set()

    def on_step(plan, t, out):
        check(plan, t, out)
        if out is not None:
            slots = [runner.bm.state_slot(r.seq) for r in plan.requests]
            assert len(set(slots)) == len(slots) and all(0 <= x < 6 for x in slots)
            slots_seen.update(slots)

    check = _checked_trace_step(runner, mirror, torch.Generator().manual_seed(7))
    runner.run(max_steps=60, on_step=on_step)
    assert max(r.num_seqs for r in runner.records) <= 6 and len(slots_seen) == 6
    assert runner.pool.check_device_errors() == 0


def test_trace_steps_match_the_oracle(cuda_dev):
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=5, out_max=40, seed=17)
    runner = TraceRunner(cuda_dev, num_blocks=300, n_steps=30, trace=trace, token_budget=1024,
                         max_chunk=256)
    mirror = Mirror(runner.pool)
    gen = torch.Generator().manual_seed(0)

    def on_step(plan, t, out):
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        rows = []
        qsl = t["qsl"].tolist()
        for i, (req, s) in enumerate(zip(plan.requests, plan.starts)):
            toks = list(range(qsl[i], qsl[i + 1]))
            if s >= req.target:                       # decode row: every head
                rows += [(toks[0], h) for h in range(runner.Hq)]
            else:                                     # chunk: first, last and a random row
                pick = {toks[0], toks[-1], toks[int(torch.randint(len(toks), (1,), generator=gen))]}
                rows += [(tk, int(torch.randint(runner.Hq, (1,), generator=gen))) for tk in pick]
        _check_rows(mirror, t, out, rows, runner.scale, f"trace step {plan.step}")
        if plan.step % 10 == 0:
            torch.cuda.synchronize()
            assert torch.equal(runner.pool.k_pool.cpu(), mirror.k)
            assert torch.equal(runner.pool.v_pool.cpu(), mirror.v)

    runner.run(max_steps=60, on_step=on_step)
    assert runner.sched.metrics["preemptions"] > 0     # the small pool forces recomputation
    assert runner.pool.check_device_errors() == 0


def test_trace_with_the_host_a_step_ahead_ends_in_the_same_pool(cuda_dev):
    # TraceRunner.step(wait=False) plans and launches step n + 1 while step n
    # runs.  The same trace run both ways (with preemption and swaps to the host
    # pool) must plan the same steps and leave both pools bit-identical, and
    # every step of the overlapped run gets its GPU time after finish().
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=20, out_max=120, seed=17)

    def run(wait):
        r = TraceRunner(cuda_dev, num_blocks=250, n_steps=30, trace=trace, token_budget=1024,
                        max_chunk=256, preempt="swap", num_host_blocks=300)
        r.run(max_steps=80, wait=wait)
        torch.cuda.synchronize()
        return r

    a, b = run(True), run(False)
    assert [(x.step, x.tokens, x.copies, x.swap_blocks) for x in a.records] == \
        [(x.step, x.tokens, x.copies, x.swap_blocks) for x in b.records]
    assert a.sched.metrics["swaps_out"] > 0 and a.sched.metrics == b.sched.metrics
    assert torch.equal(a.pool.k_pool.view(torch.int16), b.pool.k_pool.view(torch.int16))
    assert torch.equal(a.pool.v_pool.view(torch.int16), b.pool.v_pool.view(torch.int16))
    assert all(x.gpu_ms is not None and x.gpu_ms > 0 for x in b.records)
    assert a.pool.check_device_errors() == 0 and b.pool.check_device_errors() == 0


def test_recompute_reproduces_the_same_kv(cuda_dev):
    # a request preempted and re-prefilled holds bit-identical K/V afterwards
    trace = [(0, 40, 30), (0, 40, 30), (1, 40, 30)]
    runner = TraceRunner(cuda_dev, num_blocks=9, block_size=16, n_steps=200, trace=trace,
                         token_budget=256, max_chunk=64)

    def logical_kv(req):
        table = runner.bm.block_table(req.seq)
        k = runner.pool.k_pool[table].transpose(1, 2).reshape(-1, runner.Hkv, runner.d)
        return k[:req.stored].cpu()

    before = {}
    for _ in range(200):
        for r in list(runner.sched.running):
            if not r.prefilling:
                before.setdefault(r.rid, {})[r.stored] = logical_kv(r)
        if runner.step() is None and not runner.sched.has_work() and not runner.pending:
            break
        for r in list(runner.sched.running):
            if r.preemptions and not r.prefilling and r.stored in before.get(r.rid, {}):
                assert torch.equal(logical_kv(r), before[r.rid][r.stored])
                r.checked = True
    assert runner.sched.metrics["preemptions"] > 0
    assert any(getattr(r, "checked", False) for r in runner.sched.finished + runner.sched.running)


@pytest.mark.parametrize("fused", [False, True], ids=["append+attention", "one call"])
@pytest.mark.parametrize("prompt_len,bs,copies_per_prompt", [(100, 16, 3), (96, 16, 0), (37, 8, 3),
                                                              (64, 32, 0)])
def test_fork_copy_on_write(cuda_dev, prompt_len, bs, copies_per_prompt, fused):
    # fused: each decode step is one pk_paged_attention_append call after the
    # copy-on-write copies, so the new rows go where the updated tables point;
    # the mirror appends them with the manager's slots
    n_prompts, n_samples = 4, 4
    runner = ForkRunner(cuda_dev, n_prompts=n_prompts, prompt_len=prompt_len,
                        n_samples=n_samples, block_size=bs, decode_steps=6, fused=fused)
    runner.prefill()
    torch.cuda.synchronize()
    shared = runner.unique_blocks()
    assert shared == n_prompts * -(-prompt_len // bs)       # prompt blocks stored once
    # siblings read identical K/V through identical tables before any write
    for i in range(n_prompts):
        tabs = [runner.bm.block_table(runner.seqs[i * n_samples + j][0]) for j in range(n_samples)]
        assert all(t == tabs[0] for t in tabs)
    mirror = Mirror(runner.pool)
    copies = []

    def on_step(t, out):
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        rows = [(b, h) for b in range(len(runner.seqs)) for h in (0, runner.Hq - 1)]
        _check_rows(mirror, t, out, rows, runner.scale, "fork decode")
        copies.append(t["pairs"].shape[0])

    for _ in range(runner.decode_steps):
        runner.decode_step(on_step)
    torch.cuda.synchronize()
    assert torch.equal(runner.pool.k_pool.cpu(), mirror.k) and torch.equal(runner.pool.v_pool.cpu(), mirror.v)
    assert copies[0] == n_prompts * copies_per_prompt and sum(copies[1:]) == 0
    # after diverging, siblings differ only in the blocks written since the fork
    for i in range(n_prompts):
        tabs = [runner.bm.block_table(runner.seqs[i * n_samples + j][0]) for j in range(n_samples)]
        n_full = prompt_len // bs
        assert all(t[:n_full] == tabs[0][:n_full] for t in tabs)
        assert len({tuple(t[n_full:]) for t in tabs}) == n_samples
    assert runner.unique_blocks() < runner.clone_blocks()
    torch.cuda.synchronize()
    assert torch.equal(runner.pool.k_pool.cpu(), mirror.k)
    assert runner.pool.check_device_errors() == 0


def test_trace_in_swap_mode_matches_the_oracle(cuda_dev):
    # preempted requests' blocks go to a pinned host pool and come back
    # ["Batching and PagedAttention", "When blocks run out"]; attention after a
    # swap-in sees exactly the K/V written before the swap-out
    trace = trace_requests(n_steps=30, arrivals_per_step=3.0, prompt_median=256, prompt_max=1500,
                           out_min=20, out_max=120, seed=17)
    runner = TraceRunner(cuda_dev, num_blocks=250, n_steps=30, trace=trace, token_budget=1024,
                         max_chunk=256, preempt="swap", num_host_blocks=300)
    mirror = Mirror(runner.pool, runner.host)
    gen = torch.Generator().manual_seed(1)

    def on_step(plan, t, out):
        mirror.swaps(t["swaps"])
        if out is None:
            return
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        rows = []
        qsl = t["qsl"].tolist()
        for i, (req, s) in enumerate(zip(plan.requests, plan.starts)):
            toks = list(range(qsl[i], qsl[i + 1]))
            if s >= req.target or req.preemptions:    # decode rows and resumed requests: all heads
                rows += [(tk, h) for tk in {toks[0], toks[-1]} for h in range(runner.Hq)]
            else:
                pick = {toks[0], toks[-1], toks[int(torch.randint(len(toks), (1,), generator=gen))]}
                rows += [(tk, int(torch.randint(runner.Hq, (1,), generator=gen))) for tk in pick]
        _check_rows(mirror, t, out, rows, runner.scale, f"swap trace step {plan.step}")
        if plan.step % 10 == 0 or t["swaps"]:
            torch.cuda.synchronize()
            assert torch.equal(runner.pool.k_pool.cpu(), mirror.k)
            assert torch.equal(runner.pool.v_pool.cpu(), mirror.v)
            assert torch.equal(runner.host.k, mirror.hk) and torch.equal(runner.host.v, mirror.hv)

    runner.run(max_steps=60, on_step=on_step)
    m = runner.sched.metrics
    assert m["swaps_out"] > 0 and m["swaps_in"] > 0
    assert runner.pool.check_device_errors() == 0


def test_trace_with_prefix_cache_matches_the_oracle(cuda_dev):
    # requests on shared system prompts start on the prompt's blocks written by
    # an earlier request ["Batching and PagedAttention", "Sharing blocks"]:
    # attention matches the oracle, and every request's K read through its own
    # table equals, bit for bit, the values its own tokens would have
    from paged_kv_cache_chunked_b200.workloads import prefix_trace_requests, token_values
    trace = prefix_trace_requests(n_steps=30, arrivals_per_step=3.0, sys_lens=(200, 64, 320),
                                  user_median=100, user_max=800, out_min=5, out_max=40, seed=79)
    runner = TraceRunner(cuda_dev, num_blocks=500, n_steps=30, trace=trace, token_budget=1024,
                         max_chunk=256, prefix_cache=True)
    mirror = Mirror(runner.pool)
    gen = torch.Generator().manual_seed(2)

    def on_step(plan, t, out):
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        rows = []
        qsl = t["qsl"].tolist()
        for i, (req, s) in enumerate(zip(plan.requests, plan.starts)):
            toks = list(range(qsl[i], qsl[i + 1]))
            pick = {toks[0], toks[-1], toks[int(torch.randint(len(toks), (1,), generator=gen))]}
            rows += [(tk, h) for tk in pick for h in (0, runner.Hq - 1)]
        _check_rows(mirror, t, out, rows, runner.scale, f"prefix trace step {plan.step}")
        for i, req in enumerate(plan.requests):
            c = plan.context_lens[i]
            table = t["tables"][i, :-(-c // runner.bs)].long()
            got = mirror.k[table].transpose(1, 2).reshape(-1, runner.Hkv, runner.d)[:c]
            want = token_values(runner.seed, 1, runner.value_ids(req, 0, c), list(range(c)),
                                runner.Hkv, runner.d, runner.dtype)
            assert torch.equal(got, want), f"request {req.rid}: K through its table differs"

    runner.run(max_steps=60, on_step=on_step)
    st = runner.bm.stats()
    assert runner.sched.metrics["prefix_hit_tokens"] > 0 and st["prefix_hits"] > 0
    assert runner.pool.check_device_errors() == 0


@pytest.mark.parametrize("prompt_len", [1024, 1028])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_fork_workload_as_stated(cuda_dev, prompt_len, bs):
    # n-sample forks as stated: 64 prompts of 1,024 tokens (and the 1,028-token
    # variant, whose partly filled tail block is shared at every block size),
    # each forked into 4 samples sharing the prompt's blocks by reference count,
    # 32 q / 8 kv heads, head dim 128; the first 8 decode steps.  The prompt's
    # K/V is checked through every parent table, the block manager's slots,
    # copy pairs and tables step by step against the oracle manager, every
    # decode row of every step against the oracle, and the pool bit for bit at
    # the end.  Copy-on-write copies a shared block only when a write targets
    # it ["PagedAttention & Continuous Batching" (study notes),
    # "Copy-on-write"]: 1,024 tokens fill whole blocks at 8, 16 and 32, so no
    # copy; 1,028 leaves a shared tail, so 3 copies per prompt (the fourth
    # sharer writes in place), 192 in the first decode step and none after.
    from oracle import OracleBlockManager
    from paged_kv_cache_chunked_b200.workloads import token_values
    n_prompts, n_samples, steps = 64, 4, 8
    runner = ForkRunner(cuda_dev, n_prompts=n_prompts, prompt_len=prompt_len, n_samples=n_samples,
                        block_size=bs, decode_steps=steps)
    runner.prefill()
    torch.cuda.synchronize()
    # the oracle manager through the same operations
    om = OracleBlockManager(runner.num_blocks, bs)
    parents = [om.add_seq() for _ in range(n_prompts)]
    done = 0
    while done < prompt_len:
        n = min(runner.chunk, prompt_len - done)
        for p in parents:
            om.append_slots(p, n)
        done += n
    oseqs = []
    for p in parents:
        oseqs.append(p)
        oseqs += [om.fork(p) for _ in range(n_samples - 1)]
    assert [s for s, _ in runner.seqs] == oseqs
    for s in oseqs:
        assert runner.bm.block_table(s) == om.block_table(s)
    assert runner.unique_blocks() == n_prompts * -(-prompt_len // bs)
    # the prompts' K/V, read through every parent's table, is what was appended
    for i, p in enumerate(parents):
        table = torch.tensor(om.block_table(p), device=cuda_dev)
        for stream, pool in ((1, runner.pool.k_pool), (2, runner.pool.v_pool)):
            got = pool[table].transpose(1, 2).reshape(-1, runner.Hkv, runner.d)[:prompt_len]
            want = token_values(runner.seed, stream, [i * n_samples] * prompt_len, list(range(prompt_len)),
                                runner.Hkv, runner.d, runner.dtype, cuda_dev)
            assert torch.equal(got, want), f"prompt {i}"
    mirror = Mirror(runner.pool)
    copies = []

    def on_step(t, out):
        slots, pairs = [], []
        for s in oseqs:
            sl, pr = om.append_slots(s, 1)
            slots += sl
            pairs += pr
        assert t["slots"].tolist() == slots
        assert [tuple(x) for x in t["pairs"].tolist()] == pairs
        want_t = torch.full(t["tables"].shape, -1, dtype=torch.int32)
        for r, s in enumerate(oseqs):
            tab = om.block_table(s)
            want_t[r, :len(tab)] = torch.tensor(tab, dtype=torch.int32)
        assert torch.equal(t["tables"], want_t)
        mirror.apply(t["pairs"], t["k"], t["v"], t["slots"])
        _check_tokens(mirror, t, out, list(range(len(oseqs))), runner.Hq, runner.scale,
                      f"fork decode, block {bs}")
        copies.append(len(pairs))

    for _ in range(steps):
        runner.decode_step(on_step)
    want = n_prompts * (n_samples - 1) if prompt_len % bs else 0
    assert copies == [want] + [0] * (steps - 1)
    torch.cuda.synchronize()
    assert torch.equal(runner.pool.k_pool.cpu(), mirror.k)
    assert torch.equal(runner.pool.v_pool.cpu(), mirror.v)
    assert runner.pool.check_device_errors() == 0
