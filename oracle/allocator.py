"""Oracle host block manager (test infrastructure only), in plain Python.

What the pages fix:
  * the pool is a set of equal, fixed-size physical blocks; a free list holds
    the unused ones and finished requests return theirs to it
    [PagedAttention & Continuous Batching (study notes), "Block tables";
    Batching and PagedAttention, "PagedAttention", item 1];
  * each sequence has a block table of logical -> physical ids, filled left
    to right, growing by one block when the current one fills; nothing is
    reserved ahead [Batching and PagedAttention, "PagedAttention", items 2-3];
  * on a fork the child takes the parent's block ids and every shared block's
    reference count goes up; a block goes back to the pool when its count
    reaches zero; a write into a shared block first gets a fresh block and a
    copy [study notes, "Copy-on-write"; 7.8 PagedAttention & continuous
    batching (LLM deep dive), "01 Concept"];
  * allocation fails when the free list is empty [study notes, Q&A "What
    fails if you page KV but never cap concurrency?"];
  * waste is at most one partly filled block per request [Batching and
    PagedAttention, "PagedAttention"].

Readings where the pages say nothing (the GPU build's manager follows the
same ones, so block tables can be compared bit for bit):
  * free list order: first in, first out, starting as 0, 1, ..., N-1;
    allocation takes the head, a block whose count reaches zero joins the tail;
  * freeing a sequence releases its blocks from the last logical block to the
    first;
  * sequence ids count up from 0 over add_seq and fork, never reused;
  * append_slots(seq, n) first copies a shared, partly filled last block
    (the copy-on-write block is allocated before any new block), then takes
    one new block each time a token starts a block; the slot id of a token is
    physical block * block_size + offset;
  * an allocation that cannot be met in full changes nothing and counts one
    allocation failure;
  * tail waste counts every physical block in use once: block_size minus the
    slots written in it.

Swapping [Batching and PagedAttention, "When blocks run out": a preempted
request's blocks are either swapped out to CPU memory or freed and recomputed
later; all blocks of a sequence are evicted together]:
  * a host pool of equal blocks with its own free list, first in, first out
    from 0, 1, ..., H-1, like the device one;
  * swap_out(seq) moves every block of seq to the host pool at once: one host
    block per table entry, taken in logical order; the device blocks are then
    released from the last logical block to the first; the table now names
    host blocks and the sequence is "swapped";
  * swap_in(seq) does the reverse: device blocks taken in logical order, host
    blocks released last to first; the slots written in each block travel
    with it;
  * a sequence holding a shared block (count > 1) is not swapped: its blocks
    also belong to other sequences, so they cannot all leave with it (the
    caller recomputes it instead); a swap that cannot be met in full (host or
    device pool short) changes nothing;
  * a swapped sequence can only be swapped in or freed (freeing returns its
    host blocks, last to first).

Prefix cache [Batching and PagedAttention, "Sharing blocks": requests that
share a system prompt can share its blocks, the basis of prefix caching; 7.8
PagedAttention & continuous batching, "01 Concept": requests with an
identical prompt prefix can point at the same read-only blocks, and the
prefix hit rate is one of the metrics to watch]:
  * a full block of a sequence can be registered under a key that names its
    whole token prefix (positions 0 up to the block's end); the first block
    registered under a key keeps it;
  * a new sequence can start from a list of such keys: it takes, in order,
    the cached block of every key until the first key not in the cache; each
    taken block's count goes up, and the sequence starts at hits x block_size
    tokens; every key offered counts as a lookup, every block taken as a hit;
  * an entry lives while its block is referenced: when the block's count
    reaches zero it leaves the cache as the block returns to the free list
    (the pages fix no retention of unreferenced blocks).

Two pools [7.8 PagedAttention & continuous batching, "01 Concept": a hybrid
model's attention layers keep growing, paged KV while its other layers keep a
fixed-size state per sequence, so the server manages two pools with different
lifecycles]:
  * an optional pool of state slots with its own free list (first in, first
    out from 0, 1, ..., S-1): every sequence takes one slot when it is
    created (add_seq, add_seq_cached, fork) and keeps it until it is freed,
    whatever its length; KV blocks keep their on-demand lifecycle;
  * admission accounts for both pools: creating a sequence with no free slot
    fails (OracleOOM) and changes nothing; a fork's slot starts as a copy of
    the parent's state, which the caller makes;
  * a swapped-out sequence keeps its slot (only KV blocks move).
"""

from collections import deque


class OracleOOM(Exception):
    """The free list cannot supply the blocks a call needs."""


class OracleBlockManager:
    def __init__(self, num_blocks, block_size):
        if num_blocks < 0 or block_size < 1:
            raise ValueError("bad pool geometry")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_list = deque(range(num_blocks))
        self.refcount = [0] * num_blocks
        self.filled = [0] * num_blocks      # slots written in each physical block
        self.tables = {}                    # seq id -> list of physical ids
        self.lengths = {}                   # seq id -> tokens stored
        self.next_seq = 0
        self.alloc_failures = 0
        self.host_blocks = 0
        self.host_free = deque()
        self.host_filled = []
        self.swapped = set()
        self.cache = {}                     # key -> physical block
        self.key_of = {}                    # physical block -> key it is cached under
        self.prefix_lookups = 0
        self.prefix_hits = 0
        self.state_slots = 0
        self.state_free = deque()
        self.state_of = {}                  # seq id -> state slot

    # -- sequences -----------------------------------------------------
    def add_seq(self):
        if self.state_slots and not self.state_free:
            raise OracleOOM("no free state slot")
        sid = self.next_seq
        self.next_seq += 1
        self.tables[sid] = []
        self.lengths[sid] = 0
        if self.state_slots:
            self.state_of[sid] = self.state_free.popleft()
        return sid

    def set_state_slots(self, n):
        """Give every sequence a fixed-size state slot from a pool of n (once)."""
        if n < 0 or self.state_slots or self.tables:
            raise ValueError("state pool already set, negative, or sequences exist")
        self.state_slots = n
        self.state_free = deque(range(n))

    def state_slot(self, seq):
        return self.state_of.get(seq, -1)

    def _take(self):
        block = self.free_list.popleft()
        self.refcount[block] = 1
        self.filled[block] = 0
        return block

    def _release(self, block):
        self.refcount[block] -= 1
        if self.refcount[block] == 0:
            self.filled[block] = 0
            if block in self.key_of:
                del self.cache[self.key_of.pop(block)]
            self.free_list.append(block)

    def _resident(self, seq):
        if seq not in self.tables:
            raise KeyError(seq)
        if seq in self.swapped:
            raise ValueError(f"sequence {seq} is swapped out")

    def blocks_needed(self, seq, n):
        """Blocks an append of n tokens to seq would take from the free list."""
        self._resident(seq)
        length, table, bs = self.lengths[seq], self.tables[seq], self.block_size
        if n <= 0:
            return 0
        cow = 1 if (length % bs != 0 and self.refcount[table[-1]] > 1) else 0
        grow = -(-(length + n) // bs) - -(-length // bs)
        return cow + grow

    def append_slots(self, seq, n):
        """Reserve slots for the next n tokens of seq.

        Returns (slots, pairs): slot id of each new token in order, and the
        (source, destination) block pairs that must be copied before the
        tokens are written.  Raises OracleOOM with nothing changed.
        """
        self._resident(seq)
        if n < 0:
            raise ValueError("negative token count")
        if self.blocks_needed(seq, n) > len(self.free_list):
            self.alloc_failures += 1
            raise OracleOOM(seq)
        table, bs = self.tables[seq], self.block_size
        length = self.lengths[seq]
        pairs, slots = [], []
        if n > 0 and length % bs != 0 and self.refcount[table[-1]] > 1:
            src = table[-1]
            dst = self._take()
            self.filled[dst] = self.filled[src]
            self.refcount[src] -= 1
            table[-1] = dst
            pairs.append((src, dst))
        for pos in range(length, length + n):
            if pos % bs == 0:
                table.append(self._take())
            block = table[pos // bs]
            offset = pos % bs
            self.filled[block] = max(self.filled[block], offset + 1)
            slots.append(block * bs + offset)
        self.lengths[seq] = length + n
        return slots, pairs

    def append_one_each(self, seqs):
        """One token for each of seqs in order, as append_slots(seq, 1), stopping
        (without an allocation failure) at the first one whose token needs a
        block while none is free.  Returns (served, slots, pairs)."""
        slots, pairs = [], []
        for seq in seqs:
            if self.blocks_needed(seq, 1) > len(self.free_list):
                break
            s, p = self.append_slots(seq, 1)
            slots += s
            pairs += p
        return len(slots), slots, pairs

    def fork(self, parent):
        """New sequence sharing every block of parent (reference counts +1)."""
        self._resident(parent)
        if self.state_slots and not self.state_free:
            raise OracleOOM("no free state slot")
        child = self.next_seq
        self.next_seq += 1
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        if self.state_slots:
            self.state_of[child] = self.state_free.popleft()
        for block in self.tables[child]:
            self.refcount[block] += 1
        return child

    def free(self, seq):
        """Drop seq; blocks whose count reaches zero return to the free list
        (a swapped sequence returns its host blocks)."""
        table = self.tables.pop(seq)
        del self.lengths[seq]
        if seq in self.state_of:
            self.state_free.append(self.state_of.pop(seq))
        if seq in self.swapped:
            self.swapped.discard(seq)
            for h in reversed(table):
                self._release_host(h)
            return
        for block in reversed(table):
            self._release(block)

    # -- prefix cache --------------------------------------------------
    def cache_blocks(self, seq, keys):
        """Register seq's first len(keys) logical blocks (all full) under keys."""
        self._resident(seq)
        table, bs = self.tables[seq], self.block_size
        if len(keys) * bs > self.lengths[seq]:
            raise ValueError("only full blocks can be cached")
        for i, key in enumerate(keys):
            b = table[i]
            if key not in self.cache and b not in self.key_of:
                self.cache[key] = b
                self.key_of[b] = key

    def cached_prefix(self, keys):
        """Blocks a sequence starting from keys would take from the cache."""
        n = 0
        while n < len(keys) and keys[n] in self.cache:
            n += 1
        return n

    def add_seq_cached(self, keys):
        """New sequence starting on the cached blocks of keys' longest cached
        prefix.  Returns (seq id, blocks hit)."""
        sid = self.add_seq()
        hits = self.cached_prefix(keys)
        for key in keys[:hits]:
            b = self.cache[key]
            self.refcount[b] += 1
            self.tables[sid].append(b)
        self.lengths[sid] = hits * self.block_size
        self.prefix_lookups += len(keys)
        self.prefix_hits += hits
        return sid, hits

    # -- swapping ------------------------------------------------------
    def set_host_blocks(self, n):
        """Give the manager a host pool of n blocks (once)."""
        if n < 0 or self.host_blocks:
            raise ValueError("host pool already set or negative")
        self.host_blocks = n
        self.host_free = deque(range(n))
        self.host_filled = [0] * n

    def _release_host(self, h):
        self.host_filled[h] = 0
        self.host_free.append(h)

    def swap_out(self, seq):
        """Move all of seq's blocks to the host pool.  Returns the (device,
        host) block pairs to copy, in logical order.  Raises ValueError for a
        sequence that shares a block or is already swapped, OracleOOM when the
        host pool is short; nothing changes then."""
        self._resident(seq)
        table = self.tables[seq]
        if any(self.refcount[b] > 1 for b in table):
            raise ValueError(f"sequence {seq} shares blocks")
        if len(table) > len(self.host_free):
            raise OracleOOM(seq)
        pairs = []
        for b in table:
            h = self.host_free.popleft()
            self.host_filled[h] = self.filled[b]
            pairs.append((b, h))
        for b in reversed(table):
            self._release(b)
        self.tables[seq] = [h for _, h in pairs]
        self.swapped.add(seq)
        return pairs

    def swap_in(self, seq):
        """Bring a swapped sequence's blocks back to the device pool.  Returns
        the (host, device) pairs to copy, in logical order.  Raises OracleOOM
        when the device pool is short (nothing changes then)."""
        if seq not in self.swapped:
            raise ValueError(f"sequence {seq} is not swapped out")
        table = self.tables[seq]
        if len(table) > len(self.free_list):
            raise OracleOOM(seq)
        pairs = []
        for h in table:
            b = self._take()
            self.filled[b] = self.host_filled[h]
            pairs.append((h, b))
        for h in reversed(table):
            self._release_host(h)
        self.tables[seq] = [b for _, b in pairs]
        self.swapped.discard(seq)
        return pairs

    # -- views ---------------------------------------------------------
    def block_table(self, seq):
        return list(self.tables[seq])

    def length(self, seq):
        return self.lengths[seq]

    def num_free(self):
        return len(self.free_list)

    def num_used(self):
        return self.num_blocks - len(self.free_list)

    def tail_waste(self):
        """Unwritten slots summed over every physical block in use (once each)."""
        return sum(self.block_size - self.filled[b] for b in range(self.num_blocks)
                   if self.refcount[b] > 0)

    def stats(self):
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": self.num_free(),
            "used_blocks": self.num_used(),
            "alloc_failures": self.alloc_failures,
            "tail_waste_slots": self.tail_waste(),
            "num_seqs": len(self.tables),
            "host_blocks": self.host_blocks,
            "host_free_blocks": len(self.host_free),
            "prefix_lookups": self.prefix_lookups,
            "prefix_hits": self.prefix_hits,
            "cached_blocks": len(self.cache),
            "state_slots": self.state_slots,
            "state_free_slots": len(self.state_free),
        }
