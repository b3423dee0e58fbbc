// Host block manager of the paged KV cache (C ABI pk_bm_*).
//
// What it keeps, from the pages:
//  * a pool of equal physical blocks and a free list; finished requests
//    return their blocks to it ["PagedAttention & Continuous Batching"
//    (study notes), "Block tables"; "Batching and PagedAttention",
//    "PagedAttention" items 1-3: blocks are allocated one at a time on demand,
//    nothing is reserved for a maximum length];
//  * a block table per sequence, logical block i -> physical id, filled left
//    to right;
//  * reference counts: a fork copies the parent's ids and increments the
//    counts; a write into a shared block first takes a fresh block and a copy
//    of the old one (copy-on-write); a block returns to the free list when its
//    count reaches zero [study notes, "Copy-on-write"; "7.8 PagedAttention &
//    continuous batching" (LLM deep dive), "01 Concept"];
//  * allocation fails cleanly when the free list runs dry [study notes, Q&A
//    on capping concurrency], leaving the state unchanged;
//  * the operational counters the deep-dive page lists: free and used
//    blocks, allocation failures, tail waste.
//
// Swapping ["Batching and PagedAttention", "When blocks run out": a preempted
// request's blocks are swapped out to CPU memory or freed and recomputed; all
// blocks of a sequence are evicted together]: a host pool with its own FIFO
// free list; swap_out moves every block of a sequence at once (host blocks
// taken in logical order, device blocks then released last to first; the
// table then names host blocks), swap_in the reverse.  A sequence that shares
// a block is not swapped (its blocks also belong to other sequences); a swap
// that cannot be met in full changes nothing.  A swapped sequence can only be
// swapped in or freed.
//
// Prefix cache ["Batching and PagedAttention", "Sharing blocks": requests that
// share a system prompt can share its blocks, the basis of prefix caching;
// "7.8 PagedAttention & continuous batching", "01 Concept": requests with an
// identical prompt prefix point at the same read-only blocks; prefix hit rate]:
// a full block can be registered under a caller key naming its whole token
// prefix (the first registration of a key keeps it); a new sequence can start
// from a list of keys and takes, in order, the cached block of each key until
// the first miss (counts + 1, length hits x block_size; every key offered is a
// lookup, every block taken a hit); an entry lives while its block is
// referenced and leaves the cache when the block returns to the free list.
//
// Two pools ["7.8 PagedAttention & continuous batching", "01 Concept": a
// hybrid model's attention layers keep growing, paged KV while its other
// layers keep a fixed-size per-sequence state, so the server manages two pools
// with different lifecycles]: an optional pool of state slots (FIFO free list);
// every sequence takes a slot when created (add_seq, add_seq_cached, fork; a
// fork's slot is the caller's copy of the parent's state) and returns it when
// freed; creating a sequence with no free slot fails and changes nothing; a
// swapped-out sequence keeps its slot.
//
// Policy details the pages leave open, fixed so that tables are reproducible:
// FIFO free list starting as 0..N-1 (a released block joins the tail);
// a sequence's blocks are released from its last logical block to its first;
// sequence ids count up from 0; in append_slots the copy-on-write block is
// taken before any new block.
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "paged_kv.h"

namespace pk {
int fail(int code, const char *fmt, ...);
}

struct pk_bm {
    int num_blocks;
    int block_size;
    std::deque<int32_t> free_list;
    std::vector<int32_t> refcount;
    std::vector<int32_t> filled;  // slots written in each physical block
    struct Seq {
        std::vector<int32_t> table;
        int64_t len = 0;
        bool swapped = false;  // table names host blocks
        int32_t state_slot = -1;
    };
    int num_state_slots = 0;
    std::deque<int32_t> state_free;
    int num_host_blocks = 0;
    std::deque<int32_t> host_free;
    std::vector<int32_t> host_filled;
    std::unordered_map<uint64_t, int32_t> cache;   // key -> physical block
    std::unordered_map<int32_t, uint64_t> key_of;  // physical block -> its key
    int64_t prefix_lookups = 0, prefix_hits = 0;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t next_seq = 0;
    int64_t alloc_failures = 0;

    int32_t take() {
        const int32_t b = free_list.front();
        free_list.pop_front();
        refcount[b] = 1;
        filled[b] = 0;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) {
            filled[b] = 0;
            auto k = key_of.find(b);
            if (k != key_of.end()) {
                cache.erase(k->second);
                key_of.erase(k);
            }
            free_list.push_back(b);
        }
    }
    int cached_prefix(const uint64_t *keys, int n) const {
        int h = 0;
        while (h < n && cache.count(keys[h])) ++h;
        return h;
    }
    int64_t needed(const Seq &s, int n) const {
        if (n <= 0) return 0;
        const int64_t bs = block_size;
        const int cow = (s.len % bs != 0 && refcount[s.table.back()] > 1) ? 1 : 0;
        const int64_t grow = (s.len + n + bs - 1) / bs - (s.len + bs - 1) / bs;
        return cow + grow;
    }
};

using pk::fail;

namespace {
// the sequence, if it exists and is resident on the device
pk_bm::Seq *resident(pk_bm *bm, int64_t seq) {
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) {
        fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
        return nullptr;
    }
    if (it->second.swapped) {
        fail(PK_ERR_INVALID_ARG, "sequence %lld is swapped out", (long long)seq);
        return nullptr;
    }
    return &it->second;
}
const pk_bm::Seq *resident(const pk_bm *bm, int64_t seq) { return resident(const_cast<pk_bm *>(bm), seq); }
}  // namespace

extern "C" {

int pk_bm_create(int num_blocks, int block_size, pk_bm **out) {
    if (!out) return fail(PK_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (num_blocks < 0 || block_size < 1) return fail(PK_ERR_INVALID_ARG, "bad pool geometry");
    pk_bm *bm = new (std::nothrow) pk_bm();
    if (!bm) return fail(PK_ERR_INVALID_ARG, "out of host memory");
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->refcount.assign(num_blocks, 0);
    bm->filled.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) bm->free_list.push_back(b);
    *out = bm;
    return PK_OK;
}

int pk_bm_destroy(pk_bm *bm) {
    delete bm;
    return PK_OK;
}

namespace {
// a state slot for a new sequence (-1 without a state pool); false: none free
bool take_state_slot(pk_bm *bm, int32_t *slot) {
    *slot = -1;
    if (bm->num_state_slots == 0) return true;
    if (bm->state_free.empty()) return false;
    *slot = bm->state_free.front();
    bm->state_free.pop_front();
    return true;
}
}  // namespace

int pk_bm_add_seq(pk_bm *bm, int64_t *seq_out) {
    if (!bm || !seq_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    int32_t slot;
    if (!take_state_slot(bm, &slot)) return fail(PK_ERR_OOM, "no free state slot");
    const int64_t id = bm->next_seq++;
    pk_bm::Seq s;
    s.state_slot = slot;
    bm->seqs.emplace(id, std::move(s));
    *seq_out = id;
    return PK_OK;
}

int pk_bm_set_state_slots(pk_bm *bm, int num_slots) {
    if (!bm) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    if (num_slots < 0 || bm->num_state_slots != 0 || !bm->seqs.empty())
        return fail(PK_ERR_INVALID_ARG, "state pool already set, negative, or sequences exist");
    bm->num_state_slots = num_slots;
    for (int32_t i = 0; i < num_slots; ++i) bm->state_free.push_back(i);
    return PK_OK;
}

int pk_bm_state_slot(const pk_bm *bm, int64_t seq, int *slot_out) {
    if (!bm || !slot_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    *slot_out = it->second.state_slot;
    return PK_OK;
}

int pk_bm_blocks_needed(const pk_bm *bm, int64_t seq, int n, int *needed_out) {
    if (!bm || !needed_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    const pk_bm::Seq *sq = resident(bm, seq);
    if (!sq) return PK_ERR_INVALID_ARG;
    if (n < 0) return fail(PK_ERR_INVALID_ARG, "negative token count");
    *needed_out = (int)bm->needed(*sq, n);
    return PK_OK;
}

int pk_bm_append_slots(pk_bm *bm, int64_t seq, int n, int64_t *slots_out, int32_t *pairs_out,
                       int pairs_cap, int *n_pairs_out) {
    if (!bm || !n_pairs_out || (n > 0 && !slots_out)) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    pk_bm::Seq *sq = resident(bm, seq);
    if (!sq) return PK_ERR_INVALID_ARG;
    if (n < 0) return fail(PK_ERR_INVALID_ARG, "negative token count");
    pk_bm::Seq &s = *sq;
    *n_pairs_out = 0;
    if (n == 0) return PK_OK;
    const int64_t bs = bm->block_size;
    const bool cow = s.len % bs != 0 && bm->refcount[s.table.back()] > 1;
    if (cow && (pairs_cap < 1 || !pairs_out))
        return fail(PK_ERR_INVALID_ARG, "copy-on-write pair needs pairs_out");
    if (bm->needed(s, n) > (int64_t)bm->free_list.size()) {
        ++bm->alloc_failures;
        return fail(PK_ERR_OOM, "need %lld blocks, %zu free", (long long)bm->needed(s, n),
                    bm->free_list.size());
    }
    if (cow) {
        const int32_t src = s.table.back();
        const int32_t dst = bm->take();
        bm->filled[dst] = bm->filled[src];
        --bm->refcount[src];
        s.table.back() = dst;
        pairs_out[0] = src;
        pairs_out[1] = dst;
        *n_pairs_out = 1;
    }
    for (int i = 0; i < n; ++i) {
        const int64_t pos = s.len + i;
        if (pos % bs == 0) s.table.push_back(bm->take());
        const int32_t blk = s.table[pos / bs];
        const int32_t off = (int32_t)(pos % bs);
        if (bm->filled[blk] < off + 1) bm->filled[blk] = off + 1;
        slots_out[i] = (int64_t)blk * bs + off;
    }
    s.len += n;
    return PK_OK;
}

int pk_bm_append_one_each(pk_bm *bm, const int64_t *seqs, int n, int64_t *slots_out, int32_t *pairs_out,
                          int *n_pairs_out, int *n_done_out) {
    if (!bm || !n_pairs_out || !n_done_out || n < 0 || (n > 0 && (!seqs || !slots_out || !pairs_out)))
        return fail(PK_ERR_INVALID_ARG, "bad argument");
    *n_pairs_out = 0;
    *n_done_out = 0;
    for (int i = 0; i < n; ++i) {
        const pk_bm::Seq *sq = resident(bm, seqs[i]);
        if (!sq) return PK_ERR_INVALID_ARG;
        if (bm->needed(*sq, 1) > (int64_t)bm->free_list.size()) return PK_OK;  // stop: no block for it
        int np = 0;
        const int rc = pk_bm_append_slots(bm, seqs[i], 1, slots_out + i, pairs_out + 2 * *n_pairs_out, 1, &np);
        if (rc != PK_OK) return rc;
        *n_pairs_out += np;
        *n_done_out = i + 1;
    }
    return PK_OK;
}

int pk_bm_fork(pk_bm *bm, int64_t parent, int64_t *child_out) {
    if (!bm || !child_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    const pk_bm::Seq *ps = resident(bm, parent);
    if (!ps) return PK_ERR_INVALID_ARG;
    int32_t slot;
    if (!take_state_slot(bm, &slot)) return fail(PK_ERR_OOM, "no free state slot");
    pk_bm::Seq child = *ps;  // copy before emplace can rehash
    child.state_slot = slot;
    for (int32_t b : child.table) ++bm->refcount[b];
    const int64_t id = bm->next_seq++;
    bm->seqs.emplace(id, std::move(child));
    *child_out = id;
    return PK_OK;
}

int pk_bm_free(pk_bm *bm, int64_t seq) {
    if (!bm) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    const std::vector<int32_t> &t = it->second.table;
    if (it->second.state_slot >= 0) bm->state_free.push_back(it->second.state_slot);
    if (it->second.swapped) {  // its host blocks return to the host pool
        for (auto h = t.rbegin(); h != t.rend(); ++h) {
            bm->host_filled[*h] = 0;
            bm->host_free.push_back(*h);
        }
    } else {
        for (auto b = t.rbegin(); b != t.rend(); ++b) bm->release(*b);
    }
    bm->seqs.erase(it);
    return PK_OK;
}

int pk_bm_set_host_blocks(pk_bm *bm, int num_host_blocks) {
    if (!bm) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    if (num_host_blocks < 0 || bm->num_host_blocks != 0)
        return fail(PK_ERR_INVALID_ARG, "host pool already set, or negative size");
    bm->num_host_blocks = num_host_blocks;
    bm->host_filled.assign(num_host_blocks, 0);
    for (int32_t h = 0; h < num_host_blocks; ++h) bm->host_free.push_back(h);
    return PK_OK;
}

int pk_bm_swap_out(pk_bm *bm, int64_t seq, int32_t *pairs_out, int pairs_cap, int *n_pairs_out) {
    if (!bm || !n_pairs_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    *n_pairs_out = 0;
    pk_bm::Seq *sq = resident(bm, seq);
    if (!sq) return PK_ERR_INVALID_ARG;
    std::vector<int32_t> &t = sq->table;
    if ((int64_t)t.size() > pairs_cap || (!pairs_out && !t.empty()))
        return fail(PK_ERR_INVALID_ARG, "%zu pairs, capacity %d", t.size(), pairs_cap);
    for (int32_t b : t)
        if (bm->refcount[b] > 1)
            return fail(PK_ERR_UNSUPPORTED, "sequence %lld shares block %d", (long long)seq, b);
    if (t.size() > bm->host_free.size())
        return fail(PK_ERR_OOM, "need %zu host blocks, %zu free", t.size(), bm->host_free.size());
    for (size_t i = 0; i < t.size(); ++i) {
        const int32_t h = bm->host_free.front();
        bm->host_free.pop_front();
        bm->host_filled[h] = bm->filled[t[i]];
        pairs_out[2 * i] = t[i];
        pairs_out[2 * i + 1] = h;
    }
    for (auto b = t.rbegin(); b != t.rend(); ++b) bm->release(*b);
    for (size_t i = 0; i < t.size(); ++i) t[i] = pairs_out[2 * i + 1];
    sq->swapped = true;
    *n_pairs_out = (int)t.size();
    return PK_OK;
}

int pk_bm_swap_in(pk_bm *bm, int64_t seq, int32_t *pairs_out, int pairs_cap, int *n_pairs_out) {
    if (!bm || !n_pairs_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    *n_pairs_out = 0;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    pk_bm::Seq &s = it->second;
    if (!s.swapped) return fail(PK_ERR_INVALID_ARG, "sequence %lld is not swapped out", (long long)seq);
    std::vector<int32_t> &t = s.table;
    if ((int64_t)t.size() > pairs_cap || (!pairs_out && !t.empty()))
        return fail(PK_ERR_INVALID_ARG, "%zu pairs, capacity %d", t.size(), pairs_cap);
    if (t.size() > bm->free_list.size())
        return fail(PK_ERR_OOM, "need %zu blocks, %zu free", t.size(), bm->free_list.size());
    for (size_t i = 0; i < t.size(); ++i) {
        const int32_t b = bm->take();
        bm->filled[b] = bm->host_filled[t[i]];
        pairs_out[2 * i] = t[i];
        pairs_out[2 * i + 1] = b;
    }
    for (auto h = t.rbegin(); h != t.rend(); ++h) {
        bm->host_filled[*h] = 0;
        bm->host_free.push_back(*h);
    }
    for (size_t i = 0; i < t.size(); ++i) t[i] = pairs_out[2 * i + 1];
    s.swapped = false;
    *n_pairs_out = (int)t.size();
    return PK_OK;
}

int pk_bm_cache_blocks(pk_bm *bm, int64_t seq, const uint64_t *keys, int n_keys) {
    if (!bm || (n_keys > 0 && !keys) || n_keys < 0) return fail(PK_ERR_INVALID_ARG, "bad argument");
    pk_bm::Seq *sq = resident(bm, seq);
    if (!sq) return PK_ERR_INVALID_ARG;
    if ((int64_t)n_keys * bm->block_size > sq->len)
        return fail(PK_ERR_INVALID_ARG, "only full blocks can be cached (%d keys, %lld tokens)", n_keys,
                    (long long)sq->len);
    for (int i = 0; i < n_keys; ++i) {
        const int32_t b = sq->table[i];
        if (!bm->cache.count(keys[i]) && !bm->key_of.count(b)) {
            bm->cache.emplace(keys[i], b);
            bm->key_of.emplace(b, keys[i]);
        }
    }
    return PK_OK;
}

int pk_bm_cached_prefix(const pk_bm *bm, const uint64_t *keys, int n_keys, int *n_hit_out) {
    if (!bm || !n_hit_out || (n_keys > 0 && !keys) || n_keys < 0)
        return fail(PK_ERR_INVALID_ARG, "bad argument");
    *n_hit_out = bm->cached_prefix(keys, n_keys);
    return PK_OK;
}

int pk_bm_add_seq_cached(pk_bm *bm, const uint64_t *keys, int n_keys, int64_t *seq_out, int *n_hit_out) {
    if (!bm || !seq_out || !n_hit_out || (n_keys > 0 && !keys) || n_keys < 0)
        return fail(PK_ERR_INVALID_ARG, "bad argument");
    int32_t slot;
    if (!take_state_slot(bm, &slot)) return fail(PK_ERR_OOM, "no free state slot");
    const int64_t id = bm->next_seq++;
    pk_bm::Seq s;
    s.state_slot = slot;
    const int hits = bm->cached_prefix(keys, n_keys);
    for (int i = 0; i < hits; ++i) {
        const int32_t b = bm->cache.at(keys[i]);
        ++bm->refcount[b];
        s.table.push_back(b);
    }
    s.len = (int64_t)hits * bm->block_size;
    bm->seqs.emplace(id, std::move(s));
    bm->prefix_lookups += n_keys;
    bm->prefix_hits += hits;
    *seq_out = id;
    *n_hit_out = hits;
    return PK_OK;
}

int pk_bm_is_swapped(const pk_bm *bm, int64_t seq, int *swapped_out) {
    if (!bm || !swapped_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    *swapped_out = it->second.swapped ? 1 : 0;
    return PK_OK;
}

int pk_bm_block_table(const pk_bm *bm, int64_t seq, int32_t *out, int cap, int *n_out) {
    if (!bm || !n_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    const std::vector<int32_t> &t = it->second.table;
    *n_out = (int)t.size();
    if ((int)t.size() > cap || (!out && !t.empty()))
        return fail(PK_ERR_INVALID_ARG, "table of %zu entries, capacity %d", t.size(), cap);
    for (size_t i = 0; i < t.size(); ++i) out[i] = t[i];
    return PK_OK;
}

int pk_bm_fill_tables(const pk_bm *bm, const int64_t *seqs, int n_seqs, int32_t *out, int width) {
    if (!bm || (n_seqs > 0 && (!seqs || !out)) || n_seqs < 0 || width < 0)
        return fail(PK_ERR_INVALID_ARG, "bad argument");
    for (int i = 0; i < n_seqs; ++i) {
        const pk_bm::Seq *sq = resident(bm, seqs[i]);
        if (!sq) return PK_ERR_INVALID_ARG;
        const std::vector<int32_t> &t = sq->table;
        if ((int)t.size() > width)
            return fail(PK_ERR_INVALID_ARG, "table of %zu entries, width %d", t.size(), width);
        int32_t *row = out + (int64_t)i * width;
        size_t j = 0;
        for (; j < t.size(); ++j) row[j] = t[j];
        for (; j < (size_t)width; ++j) row[j] = -1;
    }
    return PK_OK;
}

int pk_bm_seq_len(const pk_bm *bm, int64_t seq, int64_t *len_out) {
    if (!bm || !len_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return fail(PK_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    *len_out = it->second.len;
    return PK_OK;
}

int pk_bm_refcount(const pk_bm *bm, int32_t block, int *count_out) {
    if (!bm || !count_out || block < 0 || block >= bm->num_blocks)
        return fail(PK_ERR_INVALID_ARG, "bad argument");
    *count_out = bm->refcount[block];
    return PK_OK;
}

int pk_bm_num_free(const pk_bm *bm, int *free_out) {
    if (!bm || !free_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    *free_out = (int)bm->free_list.size();
    return PK_OK;
}

int pk_bm_get_stats(const pk_bm *bm, pk_bm_stats *out) {
    if (!bm || !out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    out->num_blocks = bm->num_blocks;
    out->free_blocks = (int64_t)bm->free_list.size();
    out->used_blocks = bm->num_blocks - out->free_blocks;
    out->alloc_failures = bm->alloc_failures;
    int64_t waste = 0;
    for (int b = 0; b < bm->num_blocks; ++b)
        if (bm->refcount[b] > 0) waste += bm->block_size - bm->filled[b];
    out->tail_waste_slots = waste;
    out->num_seqs = (int64_t)bm->seqs.size();
    out->host_blocks = bm->num_host_blocks;
    out->host_free_blocks = (int64_t)bm->host_free.size();
    out->prefix_lookups = bm->prefix_lookups;
    out->prefix_hits = bm->prefix_hits;
    out->cached_blocks = (int64_t)bm->cache.size();
    out->state_slots = bm->num_state_slots;
    out->state_free_slots = (int64_t)bm->state_free.size();
    return PK_OK;
}

}  // extern "C"
