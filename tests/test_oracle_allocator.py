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
    referenced = {}
    for sid, table in bm.tables.items():
        assert len(table) == -(-bm.lengths[sid] // bm.block_size)
        for b in table:
            referenced[b] = referenced.get(b, 0) + 1
    # a block is in the pool or referenced, never both, never neither
    assert bm.num_free() + len(referenced) == bm.num_blocks
    assert set(bm.free_list).isdisjoint(referenced)
    for b in range(bm.num_blocks):
        assert bm.refcount[b] == referenced.get(b, 0)
    # at most one partly filled block per sequence
    assert bm.tail_waste() <= (bm.block_size - 1) * len(bm.tables)


@pytest.mark.parametrize("seed", range(5))
def test_random_operation_sequences_keep_invariants(seed):
    rng = random.Random(seed)
    bm = OracleBlockManager(40, rng.choice([1, 4, 16]))
    live = []
    for _ in range(400):
        op = rng.random()
        if op < 0.2 or not live:
            live.append(bm.add_seq())
        elif op < 0.35:
            live.append(bm.fork(rng.choice(live)))
        elif op < 0.5:
            s = rng.choice(live)
            live.remove(s)
            bm.free(s)
        else:
            s = rng.choice(live)
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
