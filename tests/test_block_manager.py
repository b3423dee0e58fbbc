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
                          "host_blocks": ob.host_blocks, "host_free_blocks": len(ob.host_free)}
    for sid in ob.tables:
        assert bm.block_table(sid) == ob.block_table(sid)
        assert bm.length(sid) == ob.length(sid)
        assert bm.is_swapped(sid) == (sid in ob.swapped)
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
    for step in range(500):
        op = rng.random()
        resident = [s for s in live if s not in ob.swapped]
        if op < 0.15 or not resident:
            a, b = bm.add_seq(), ob.add_seq()
            assert a == b
            live.append(a)
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
