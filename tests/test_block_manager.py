"""The C++ block manager (pk_bm_* through the C ABI) against the oracle
block manager: identical tables, slots, copy pairs, reference counts and
counters, operation by operation.  Host-only, no GPU."""

import random

import pytest

from oracle import OracleBlockManager, OracleOOM, capacity
from paged_kv_cache_chunked_b200.api import BlockManager
from paged_kv_cache_chunked_b200._lib import OutOfBlocks, PagedKVError
from paged_kv_cache_chunked_b200.workloads import page_toy_lengths


def _same_state(bm, ob):
    assert bm.stats() == {"num_blocks": ob.num_blocks, "free_blocks": ob.num_free(),
                          "used_blocks": ob.num_used(), "alloc_failures": ob.alloc_failures,
                          "tail_waste_slots": ob.tail_waste(), "num_seqs": len(ob.tables),
                          "host_blocks": ob.host_blocks, "host_free_blocks": len(ob.host_free),
                          "prefix_lookups": ob.prefix_lookups, "prefix_hits": ob.prefix_hits,
                          "cached_blocks": len(ob.cache), "state_slots": ob.state_slots,
                          "state_free_slots": len(ob.state_free)}
    for sid in ob.tables:
        assert bm.block_table(sid) == ob.block_table(sid)
        assert bm.length(sid) == ob.length(sid)
        assert bm.is_swapped(sid) == (sid in ob.swapped)
        assert bm.state_slot(sid) == ob.state_slot(sid)
    for b in range(ob.num_blocks):
        assert bm.refcount(b) == ob.refcount[b]


@pytest.mark.parametrize("seed", range(6))
def test_random_operations_match_the_oracle(seed):
    rng = random.Random(100 + seed)
    nb, bs = rng.choice([(24, 4), (64, 16), (40, 1), (30, 8)])
    bm, ob = BlockManager(nb, bs), OracleBlockManager(nb, bs)
    bm.set_host_blocks(nb // 2)
    ob.set_host_blocks(nb // 2)
    live = []
    prompt_keys = {}
    for step in range(500):
        op = rng.random()
        resident = [s for s in live if s not in ob.swapped]
        if op < 0.08 or not resident:
            a, b = bm.add_seq(), ob.add_seq()
            assert a == b
            live.append(a)
        elif op < 0.15:
            # a request on one of three shared prompts (keys name prefixes)
            g = rng.randrange(3)
            keys = [1000 * g + i for i in range(rng.randint(0, 4))]
            assert bm.cached_prefix(keys) == ob.cached_prefix(keys)
            a, b = bm.add_seq_cached(keys), ob.add_seq_cached(keys)
            assert a == b
            live.append(a[0])
            prompt_keys[a[0]] = keys
        elif op < 0.24 and any(s in prompt_keys for s in resident):
            s = rng.choice([s for s in resident if s in prompt_keys])
            full = min(len(prompt_keys[s]), ob.length(s) // bs)
            bm.cache_blocks(s, prompt_keys[s][:full])
            ob.cache_blocks(s, prompt_keys[s][:full])
        elif op < 0.25:
            p = rng.choice(resident)
            a, b = bm.fork(p), ob.fork(p)
            assert a == b
            live.append(a)
        elif op < 0.4:
            s = rng.choice(live)
            live.remove(s)
            bm.free(s)
            ob.free(s)
        elif op < 0.5:
            # swap out or back in; refusals must match: a shared block
            # (PK_ERR_UNSUPPORTED), a pool short of blocks (PK_ERR_OOM)
            s = rng.choice(live)
            ours, theirs = (bm.swap_in, ob.swap_in) if s in ob.swapped else (bm.swap_out, ob.swap_out)
            try:
                ref = theirs(s)
            except OracleOOM:
                with pytest.raises(OutOfBlocks):
                    ours(s)
            except ValueError:
                with pytest.raises(PagedKVError) as e:
                    ours(s)
                assert e.value.code == 3
            else:
                assert ours(s) == ref
        elif op < 0.6:
            # one token each for a few sequences, stopping where a block is missing
            seqs = rng.sample(resident, min(len(resident), rng.randint(1, 6)))
            assert bm.append_one_each(seqs) == ob.append_one_each(seqs)
        else:
            s = rng.choice(resident)
            n = rng.randint(0, 3 * bs)
            assert bm.blocks_needed(s, n) == ob.blocks_needed(s, n)
            try:
                ref = ob.append_slots(s, n)
            except OracleOOM:
                with pytest.raises(OutOfBlocks):
                    bm.append_slots(s, n)
            else:
                assert bm.append_slots(s, n) == (ref[0], ref[1])
        if step % 25 == 0:
            _same_state(bm, ob)
    _same_state(bm, ob)


def test_prefix_cache_script_matches_the_oracle():
    # requests on two shared prompts arrive, hit, finish and come back, in
    # both managers, state compared after every call
    bm, ob = BlockManager(64, 4), OracleBlockManager(64, 4)
    keys = {g: [100 * g + i for i in range(5)] for g in (1, 2)}
    live = {}
    script = [("new", 1, 18), ("new", 2, 9), ("reg", 0), ("reg", 1), ("new", 1, 22), ("new", 2, 12),
              ("new", 1, 7), ("free", 0), ("new", 1, 30), ("reg", 4), ("free", 2), ("free", 4),
              ("new", 1, 20), ("free", 6), ("free", 5), ("new", 1, 20), ("new", 2, 5)]
    for i, step in enumerate(script):
        if step[0] == "new":
            _, g, n = step
            a, b = bm.add_seq_cached(keys[g]), ob.add_seq_cached(keys[g])
            assert a == b
            live[len(live)] = (a[0], g)
            ref = ob.append_slots(a[0], n)
            assert bm.append_slots(a[0], n) == (ref[0], ref[1])
        elif step[0] == "reg":
            s_, g = live[step[1]]
            full = min(len(keys[g]), ob.length(s_) // 4)
            bm.cache_blocks(s_, keys[g][:full])
            ob.cache_blocks(s_, keys[g][:full])
        else:
            s_, _ = live[step[1]]
            bm.free(s_)
            ob.free(s_)
        _same_state(bm, ob)
    st = bm.stats()
    assert st["prefix_hits"] == 20 and st["prefix_lookups"] == 5 * 9


@pytest.mark.parametrize("seed", range(3))
def test_two_pool_operations_match_the_oracle(seed):
    # with a pool of state slots, sequence creation and fork fail cleanly when
    # no slot is free; slots follow sequences in both managers
    rng = random.Random(300 + seed)
    bm, ob = BlockManager(48, 8), OracleBlockManager(48, 8)
    bm.set_state_slots(5)
    ob.set_state_slots(5)
    live = []
    for step in range(300):
        op = rng.random()
        if op < 0.25 or not live:
            try:
                b = ob.add_seq()
            except OracleOOM:
                with pytest.raises(OutOfBlocks):
                    bm.add_seq()
                continue
            assert bm.add_seq() == b
            live.append(b)
        elif op < 0.4:
            p = rng.choice(live)
            try:
                b = ob.fork(p)
            except OracleOOM:
                with pytest.raises(OutOfBlocks):
                    bm.fork(p)
                continue
            assert bm.fork(p) == b
            live.append(b)
        elif op < 0.6:
            s_ = rng.choice(live)
            live.remove(s_)
            bm.free(s_)
            ob.free(s_)
        else:
            s_ = rng.choice(live)
            n = rng.randint(0, 20)
            try:
                ref = ob.append_slots(s_, n)
            except OracleOOM:
                with pytest.raises(OutOfBlocks):
                    bm.append_slots(s_, n)
            else:
                assert bm.append_slots(s_, n) == (ref[0], ref[1])
        _same_state(bm, ob)
        assert len(live) <= 5


def test_page_toy_capacity_through_the_product_manager():
    # "Batching and PagedAttention", "Try it": 60 requests admitted, 98.6%
    lengths = page_toy_lengths()
    bm = BlockManager(32768 // 16, 16)
    n = 0
    for L in lengths:
        s = bm.add_seq()
        try:
            bm.append_slots(s, L)
        except OutOfBlocks:
            bm.free(s)
            break
        n += 1
    assert n == 60
    assert round(100 * sum(lengths[:n]) / (bm.num_used() * 16), 1) == 98.6
    assert capacity.admit_paged(lengths, 32768, 16)[0] == n


def test_fill_tables_pads_with_minus_one():
    bm = BlockManager(16, 4)
    a, b = bm.add_seq(), bm.add_seq()
    bm.append_slots(a, 9)
    bm.append_slots(b, 1)
    t = bm.fill_tables([b, a], 4)
    assert t.tolist() == [bm.block_table(b) + [-1, -1, -1], bm.block_table(a) + [-1]]
