"""Pins for the oracle block manager and the capacity arithmetic (CPU only).

Pinned to the pages' worked examples (tests/golden/, each with its citation)
and to invariants the pages state: a block returns to the pool when no table
references it, a shared prefix is stored once until a write, and waste is at
most one partly filled block per sequence.
"""

import json
import os
import random

import pytest

from oracle import OracleBlockManager, OracleOOM, capacity
from paged_kv_cache_chunked_b200.workloads import page_toy_lengths

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_page_toy_capacity():
    gold = _golden("page_toy_capacity.json")
    lengths = page_toy_lengths()
    n, used, real = capacity.admit_reserve_max(lengths, gold["capacity_slots"], gold["max_len"])
    assert n == gold["reserve_max"]["admitted"]
    assert round(100 * real / used, 1) == gold["reserve_max"]["real_pct"]
    n, used, real = capacity.admit_paged(lengths, gold["capacity_slots"], gold["block_size"])
    assert n == gold["paged"]["admitted"]
    assert round(100 * real / used, 1) == gold["paged"]["real_pct"]
    assert round(capacity.mean_tail_waste(lengths, gold["block_size"]), 1) == \
        gold["mean_tail_waste_slots"]


def test_toy_block_table_sandbox():
    gold = _golden("toy_block_table.json")
    bm = OracleBlockManager(8, gold["block_size"])
    s = bm.add_seq()
    slots, pairs = bm.append_slots(s, gold["tokens"])
    assert len(bm.block_table(s)) == gold["blocks"] and pairs == []
    assert slots == [bm.block_table(s)[i // 4] * 4 + i % 4 for i in range(10)]
    child = bm.fork(s)
    assert bm.block_table(child) == bm.block_table(s)
    assert all(bm.refcount[b] == gold["refcount_after_fork"] for b in bm.block_table(s))
    assert bm.num_used() == gold["blocks"]


def test_pitfall_beam_fork():
    gold = _golden("pitfall_beam.json")
    bm = OracleBlockManager(64, gold["block_size"])
    s = bm.add_seq()
    bm.append_slots(s, gold["tokens"])
    assert len(bm.block_table(s)) == gold["blocks"]
    assert bm.tail_waste() == gold["internal_fragmentation_slots"]
    for _ in range(gold["beam_width"] - 1):
        bm.fork(s)
    assert bm.num_used() == gold["physical_blocks_copy_on_write"]
    # a full clone gives every beam private copies of every block
    clone = OracleBlockManager(64, gold["block_size"])
    for _ in range(gold["beam_width"]):
        clone.append_slots(clone.add_seq(), gold["tokens"])
    assert clone.num_used() == gold["physical_blocks_full_clone"]


def test_hybrid_capacity_arithmetic():
    gold = _golden("hybrid_capacity.json")
    per_tok = gold["kv_bytes_per_token"]
    # the long-document workload's geometry (4 kv heads x 256 dims, bf16, per
    # layer) reproduces the page's per-token bill over 16 attention layers
    assert capacity.kv_bytes_per_token(gold["attention_layers"], 4, 256, 2) == per_tok
    assert gold["native_context"] * per_tok == gold["bytes_per_sequence_at_native_context"]
    assert capacity.block_bytes(gold["block_tokens"], per_tok) == gold["block_bytes"]
    assert gold["session_tokens"] * per_tok == gold["session_kv_bytes"]
    mib = 1 << 20
    assert (gold["session_kv_bytes"] + gold["fixed_state_mib"] * mib) // mib == gold["session_mib"]
    assert capacity.sessions_in_pool(gold["pool_mib"] * mib, gold["session_tokens"], per_tok,
                                     gold["fixed_state_mib"] * mib) == gold["paged_sessions"]
    assert gold["pool_mib"] * mib // gold["bytes_per_sequence_at_native_context"] == \
        gold["reserved_sessions"]


def test_copy_on_write_first_write_into_shared_tail():
    bm = OracleBlockManager(16, 4)
    p = bm.add_seq()
    bm.append_slots(p, 6)                      # blocks [0, 1]; block 1 holds 2 tokens
    c = bm.fork(p)
    slots, pairs = bm.append_slots(c, 1)       # child writes into the shared tail
    assert pairs == [(1, 2)]
    assert bm.block_table(c) == [0, 2] and bm.block_table(p) == [0, 1]
    assert slots == [2 * 4 + 2]
    assert bm.refcount[0] == 2 and bm.refcount[1] == 1 and bm.refcount[2] == 1
    slots, pairs = bm.append_slots(p, 1)       # parent is now the only owner: in place
    assert pairs == [] and slots == [1 * 4 + 2]


def test_full_shared_blocks_are_never_copied():
    bm = OracleBlockManager(16, 4)
    p = bm.add_seq()
    bm.append_slots(p, 8)                      # two full blocks
    c = bm.fork(p)
    slots, pairs = bm.append_slots(c, 1)       # next token starts a fresh block
    assert pairs == [] and bm.block_table(c)[:2] == bm.block_table(p)


def test_oom_changes_nothing():
    bm = OracleBlockManager(3, 4)
    s = bm.add_seq()
    bm.append_slots(s, 9)
    before = (list(bm.free_list), list(bm.refcount), bm.block_table(s), bm.length(s))
    with pytest.raises(OracleOOM):
        bm.append_slots(s, 4)
    assert (list(bm.free_list), list(bm.refcount), bm.block_table(s), bm.length(s)) == before
    assert bm.alloc_failures == 1
    bm.free(s)
    assert bm.num_free() == 3


def _check_invariants(bm):
    referenced, host_referenced = {}, set()
    for sid, table in bm.tables.items():
        assert len(table) == -(-bm.lengths[sid] // bm.block_size)
        if sid in bm.swapped:           # a swapped table names host blocks, each once
            assert host_referenced.isdisjoint(table) and len(set(table)) == len(table)
            host_referenced.update(table)
            continue
        for b in table:
            referenced[b] = referenced.get(b, 0) + 1
    # a block is in the pool or referenced, never both, never neither
    assert bm.num_free() + len(referenced) == bm.num_blocks
    assert set(bm.free_list).isdisjoint(referenced)
    for b in range(bm.num_blocks):
        assert bm.refcount[b] == referenced.get(b, 0)
    # the same for the host pool
    assert len(bm.host_free) + len(host_referenced) == bm.host_blocks
    assert set(bm.host_free).isdisjoint(host_referenced)
    # at most one partly filled block per sequence on the device
    assert bm.tail_waste() <= (bm.block_size - 1) * (len(bm.tables) - len(bm.swapped))


@pytest.mark.parametrize("seed", range(5))
def test_random_operation_sequences_keep_invariants(seed):
    rng = random.Random(seed)
    bm = OracleBlockManager(40, rng.choice([1, 4, 16]))
    bm.set_host_blocks(30)
    live = []
    for _ in range(400):
        op = rng.random()
        resident = [s for s in live if s not in bm.swapped]
        if op < 0.2 or not resident:
            live.append(bm.add_seq())
        elif op < 0.3:
            live.append(bm.fork(rng.choice(resident)))
        elif op < 0.45:
            s = rng.choice(live)
            live.remove(s)
            bm.free(s)
        elif op < 0.55:
            s = rng.choice(live)
            try:
                if s in bm.swapped:
                    table = bm.block_table(s)
                    pairs = bm.swap_in(s)
                    assert [h for h, _ in pairs] == table and bm.block_table(s) == [d for _, d in pairs]
                else:
                    table = bm.block_table(s)
                    pairs = bm.swap_out(s)
                    assert [d for d, _ in pairs] == table and bm.block_table(s) == [h for _, h in pairs]
            except (OracleOOM, ValueError):
                pass
        else:
            s = rng.choice(resident)
            shared_tail = (bm.length(s) % bm.block_size != 0
                           and bm.refcount[bm.block_table(s)[-1]] > 1)
            try:
                slots, pairs = bm.append_slots(s, rng.randint(0, 20))
            except OracleOOM:
                continue
            assert len(pairs) == (1 if shared_tail and slots else 0)
            assert len(set(slots)) == len(slots)
        _check_invariants(bm)
    for s in live:
        bm.free(s)
    assert bm.num_free() == bm.num_blocks


def test_swap_round_trip_restores_every_sequence_kv():
    # "a preempted request's blocks are either swapped out to CPU memory or
    # freed and recomputed" [Batching and PagedAttention, "When blocks run
    # out"]: after swap-out, reuse of the freed device blocks by another
    # sequence, and swap-in, both sequences read back exactly what they wrote
    import torch
    import oracle
    bs, H, d = 4, 2, 3
    bm = OracleBlockManager(6, bs)
    bm.set_host_blocks(4)
    kp, vp = torch.zeros(6, H, bs, d), torch.zeros(6, H, bs, d)
    hk, hv = torch.full((4, H, bs, d), float("nan")), torch.full((4, H, bs, d), float("nan"))
    written = {}

    def write(seq, n, base):
        slots, pairs = bm.append_slots(seq, n)
        assert pairs == []
        k = base + torch.arange(n * H * d, dtype=torch.float32).reshape(n, H, d)
        oracle.kv_append(kp, vp, k, -k, torch.tensor(slots))
        written.setdefault(seq, []).append(k)

    def logical(seq):
        t = torch.tensor(bm.block_table(seq))
        n = bm.length(seq)
        return (kp[t].transpose(1, 2).reshape(-1, H, d)[:n], vp[t].transpose(1, 2).reshape(-1, H, d)[:n])

    a, b = bm.add_seq(), bm.add_seq()
    write(a, 10, 0.0)                         # blocks 0, 1, 2
    write(b, 5, 1000.0)                       # blocks 3, 4
    before_a = logical(a)
    oracle.swap_blocks(kp, vp, hk, hv, bm.swap_out(a), to_host=True)
    assert bm.num_free() == 4 and bm.stats()["host_free_blocks"] == 1
    c = bm.add_seq()
    write(c, 8, 5000.0)                       # takes block 5 and a's old block 2, overwriting it
    assert 2 in bm.block_table(c)
    bm.free(c)
    oracle.swap_blocks(kp, vp, hk, hv, bm.swap_in(a), to_host=False)
    assert bm.block_table(a) != [0, 1, 2]      # a lands on other physical blocks
    for got, want in zip(logical(a), before_a):
        assert torch.equal(got, want)
    kb = torch.cat(written[b])
    assert torch.equal(logical(b)[0], kb) and torch.equal(logical(b)[1], -kb)
    assert bm.stats()["host_free_blocks"] == 4
    _check_invariants(bm)


def test_swap_refusals_change_nothing():
    bm = OracleBlockManager(8, 4)
    bm.set_host_blocks(2)
    s = bm.add_seq()
    bm.append_slots(s, 9)                      # 3 blocks
    c = bm.fork(s)
    state = lambda: (list(bm.free_list), list(bm.refcount), list(bm.host_free), bm.block_table(s),
                     set(bm.swapped))
    before = state()
    with pytest.raises(ValueError):            # shares blocks with its fork
        bm.swap_out(s)
    assert state() == before
    bm.free(c)
    before = state()
    with pytest.raises(OracleOOM):             # 3 blocks, 2 host blocks
        bm.swap_out(s)
    assert state() == before
    with pytest.raises(ValueError):            # not swapped
        bm.swap_in(s)
    t = bm.add_seq()
    bm.append_slots(t, 4)
    big = OracleBlockManager(3, 4)
    big.set_host_blocks(3)
    u = big.add_seq()
    big.append_slots(u, 12)                    # 3 blocks, pool full
    big.swap_out(u)
    v = big.add_seq()
    big.append_slots(v, 1)                     # the device pool now has 2 free blocks
    before = (list(big.free_list), list(big.host_free), big.block_table(u))
    with pytest.raises(OracleOOM):
        big.swap_in(u)
    assert (list(big.free_list), list(big.host_free), big.block_table(u)) == before
    with pytest.raises(ValueError):            # a swapped sequence takes no appends
        big.append_slots(u, 1)
    big.free(u)                                # returns its host blocks
    assert big.stats()["host_free_blocks"] == 3


# ---------------------------------------------------------------- prefix cache
def test_prefix_cache_shares_a_system_prompt_across_requests():
    # "requests that share a system prompt can share its blocks too, which is
    # the basis of prefix caching" [Batching and PagedAttention, "Sharing
    # blocks"]: the second request reads the first one's prompt blocks, which
    # were written once, and writes only its own suffix
    import torch
    import oracle
    bs, H, d = 16, 2, 4
    bm = OracleBlockManager(12, bs)
    kp, vp = torch.zeros(12, H, bs, d), torch.zeros(12, H, bs, d)
    keys = ["sys0", "sys1"]                        # two full blocks of system prompt
    sys_k = torch.randn(32, H, d)

    a, hits = bm.add_seq_cached(keys)
    assert hits == 0 and bm.length(a) == 0
    slots, _ = bm.append_slots(a, 40)             # system prompt + 8 own tokens
    oracle.kv_append(kp, vp, torch.cat([sys_k, torch.randn(8, H, d)]), torch.zeros(40, H, d),
                     torch.tensor(slots))
    bm.cache_blocks(a, keys)
    b, hits = bm.add_seq_cached(keys + ["b-own"])
    assert hits == 2 and bm.length(b) == 32
    assert bm.block_table(b) == bm.block_table(a)[:2]
    assert [bm.refcount[x] for x in bm.block_table(b)] == [2, 2]
    slots, pairs = bm.append_slots(b, 5)          # b's suffix starts a block of its own
    assert pairs == [] and all(s // bs not in bm.block_table(a) for s in slots)
    t = torch.tensor(bm.block_table(b))
    got = kp[t].transpose(1, 2).reshape(-1, H, d)[:32]
    assert torch.equal(got, sys_k)
    assert bm.stats()["prefix_lookups"] == 5 and bm.stats()["prefix_hits"] == 2
    _check_invariants(bm)


def test_prefix_cache_entries_live_while_referenced():
    bm = OracleBlockManager(8, 4)
    a, _ = bm.add_seq_cached(["k0", "k1"])
    bm.append_slots(a, 8)
    bm.cache_blocks(a, ["k0", "k1"])
    b, hits = bm.add_seq_cached(["k0", "k1"])
    assert hits == 2
    bm.free(a)                                     # b still references both blocks
    assert bm.cached_prefix(["k0", "k1"]) == 2
    bm.free(b)                                     # counts reach zero: entries leave
    assert bm.cached_prefix(["k0"]) == 0 and bm.stats()["cached_blocks"] == 0
    assert bm.num_free() == 8


def test_prefix_cache_first_registration_wins_and_needs_full_blocks():
    bm = OracleBlockManager(8, 4)
    a, _ = bm.add_seq_cached([])
    bm.append_slots(a, 6)
    with pytest.raises(ValueError):
        bm.cache_blocks(a, ["x0", "x1"])           # block 1 holds 2 of 4 slots
    bm.cache_blocks(a, ["x0"])
    b, _ = bm.add_seq_cached([])
    bm.append_slots(b, 4)
    bm.cache_blocks(b, ["x0"])                     # already cached: a's block keeps it
    c, hits = bm.add_seq_cached(["x0"])
    assert hits == 1 and bm.block_table(c) == [bm.block_table(a)[0]]
    _check_invariants(bm)


@pytest.mark.parametrize("seed", range(3))
def test_random_operations_with_prefix_cache_keep_invariants(seed):
    rng = random.Random(50 + seed)
    bs = rng.choice([4, 16])
    bm = OracleBlockManager(60, bs)
    live = []
    for _ in range(400):
        op = rng.random()
        if op < 0.25 or not live:
            g = rng.randrange(3)                    # one of three shared prompts
            keys = [f"g{g}b{i}" for i in range(rng.randint(0, 4))]
            s, hits = bm.add_seq_cached(keys)
            assert bm.length(s) == hits * bs
            live.append((s, keys))
        elif op < 0.4:
            s, keys = rng.choice(live)
            full = min(len(keys), bm.length(s) // bs)
            bm.cache_blocks(s, keys[:full])
        elif op < 0.55:
            item = rng.choice(live)
            live.remove(item)
            bm.free(item[0])
        else:
            s, _ = rng.choice(live)
            try:
                bm.append_slots(s, rng.randint(0, 3 * bs))
            except OracleOOM:
                pass
        _check_invariants(bm)
        for key, b in bm.cache.items():             # cached blocks are referenced and full
            assert bm.refcount[b] > 0 and bm.filled[b] == bs
    for s, _ in live:
        bm.free(s)
    assert bm.num_free() == 60 and bm.stats()["cached_blocks"] == 0


# ---------------------------------------------------------------- two pools
def test_two_pools_hold_the_pages_ten_long_document_sessions():
    # [7.8 PagedAttention & continuous batching, "01 Concept"]: 32,768-token
    # sessions at 64 KiB of KV per token (2,048 one-MiB blocks of 16 tokens)
    # plus a 144 MiB per-sequence state, in a 23,859 MiB pool: ten sessions.
    # Split as ten state slots and the rest in KV blocks, all ten fit and grow
    # to full length, and an eleventh finds no state slot; with eleven slots
    # the KV pool is too small for eleven full sessions.
    gold = capacity.sessions_in_pool(23_859, 32_768, 64 / 1024, 144)
    assert gold == 10
    bm = OracleBlockManager(23_859 - 10 * 144, 16)
    bm.set_state_slots(10)
    seqs = [bm.add_seq() for _ in range(10)]
    for s in seqs:
        bm.append_slots(s, 32_768)
    assert sorted(bm.state_slot(s) for s in seqs) == list(range(10))
    with pytest.raises(OracleOOM):
        bm.add_seq()
    assert bm.stats()["num_seqs"] == 10
    bm11 = OracleBlockManager(23_859 - 11 * 144, 16)
    bm11.set_state_slots(11)
    grown = 0
    for _ in range(11):
        s = bm11.add_seq()
        try:
            bm11.append_slots(s, 32_768)
            grown += 1
        except OracleOOM:
            pass
    assert grown == 10


def test_state_slots_follow_sequence_lifetimes():
    bm = OracleBlockManager(16, 4)
    bm.set_state_slots(3)
    a = bm.add_seq()
    bm.append_slots(a, 9)
    c = bm.fork(a)                                  # a fork takes its own slot
    assert bm.state_slot(a) != bm.state_slot(c)
    b, _ = bm.add_seq_cached([])
    assert bm.stats()["state_free_slots"] == 0
    before = (list(bm.free_list), dict(bm.tables), bm.next_seq)
    with pytest.raises(OracleOOM):
        bm.fork(a)
    with pytest.raises(OracleOOM):
        bm.add_seq_cached(["k"])
    assert (list(bm.free_list), dict(bm.tables), bm.next_seq) == before
    assert bm.stats()["prefix_lookups"] == 0
    bm.free(a)                                      # the slot returns, whatever the length
    d = bm.add_seq()
    assert bm.state_slot(d) == 0 and bm.stats()["state_free_slots"] == 0
    bm.set_host_blocks(8)
    bm.append_slots(b, 4)
    bm.swap_out(b)                                  # a swapped sequence keeps its slot
    assert bm.state_slot(b) >= 0 and bm.stats()["state_free_slots"] == 0


# ---------------------------------------------------------------- one token for each decode
def test_append_one_each_worked_example():
    # four 4-slot blocks, FIFO free list 0..3.  A holds a full block, B two
    # tokens, C three: one free block left.  Worked by hand from the table rule
    # ["PagedAttention & Continuous Batching" (study notes), "Block tables":
    # position p lives in logical block p // bs at offset p % bs; a new block is
    # taken only when a token starts one].
    bm = OracleBlockManager(4, 4)
    a, b, c = bm.add_seq(), bm.add_seq(), bm.add_seq()
    assert bm.append_slots(a, 4) == ([0, 1, 2, 3], [])
    assert bm.append_slots(b, 2) == ([4, 5], [])
    assert bm.append_slots(c, 3) == ([8, 9, 10], [])
    # B at position 2 (block 1, offset 2), C at 3 (block 2, offset 3), A at 4
    # starts a block (the free block 3), A at 5 fills it
    assert bm.append_one_each([b, c, a, a]) == (4, [6, 11, 12, 13], [])
    assert bm.num_free() == 0
    # A at 6 and B at 3 fit; C at 4 needs a block and none is free: the call
    # stops there, counts no allocation failure and leaves C and A's second
    # request alone
    assert bm.append_one_each([a, b, c, a]) == (2, [14, 7], [])
    assert bm.alloc_failures == 0
    assert (bm.length(a), bm.length(b), bm.length(c)) == (7, 4, 4)
    assert bm.block_table(c) == [2] and bm.block_table(a) == [0, 3]


def test_append_one_each_copy_on_write_and_stop():
    # a fork shares a partly filled block: the first sharer to write copies it
    # into a fresh block ["PagedAttention & Continuous Batching" (study notes),
    # "Copy-on-write"], the last one writes in place; with no block left for a
    # copy the call stops before that sequence
    bm = OracleBlockManager(3, 4)
    p = bm.add_seq()
    bm.append_slots(p, 6)                       # blocks 0, 1; block 1 holds 2 tokens
    d = bm.fork(p)
    assert bm.append_one_each([d, p]) == (2, [10, 6], [(1, 2)])
    assert bm.block_table(d) == [0, 2] and bm.block_table(p) == [0, 1]
    e = bm.fork(p)                              # block 1 shared again, 3 tokens in it
    assert bm.append_one_each([e, p]) == (0, [], [])
    assert bm.alloc_failures == 0
    assert bm.block_table(e) == [0, 1] and bm.refcount[1] == 2 and bm.length(e) == 7


def test_append_one_each_equals_single_appends_until_the_first_refusal():
    # the same tokens one append_slots(seq, 1) at a time: identical slots, pairs
    # and state up to the first append that would be refused; nothing after it
    import copy
    rng = random.Random(11)
    for trial in range(40):
        bm = OracleBlockManager(rng.randint(6, 30), rng.choice([2, 4, 8]))
        seqs = []
        for _ in range(rng.randint(1, 6)):
            s = bm.add_seq()
            seqs.append(s)
            n = rng.randint(0, 3 * bm.block_size)
            if bm.blocks_needed(s, n) <= bm.num_free():
                bm.append_slots(s, n)
        for _ in range(rng.randint(0, 3)):
            seqs.append(bm.fork(rng.choice(seqs)))
        order = [rng.choice(seqs) for _ in range(rng.randint(1, 12))]
        ref = copy.deepcopy(bm)
        slots, pairs, served = [], [], 0
        for s in order:
            failures = ref.alloc_failures
            try:
                sl, pr = ref.append_slots(s, 1)
            except OracleOOM:
                ref.alloc_failures = failures     # the refused append is not part of the call
                break
            slots += sl
            pairs += pr
            served += 1
        assert bm.append_one_each(order) == (served, slots, pairs), trial
        assert bm.tables == ref.tables and bm.lengths == ref.lengths
        assert bm.refcount == ref.refcount and list(bm.free_list) == list(ref.free_list)
        assert bm.alloc_failures == ref.alloc_failures
