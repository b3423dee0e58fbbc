// Host side of the tensor-core attention path: workspace layout and the
// dispatch of a call.  With at most 8 q heads per kv head, the one-token
// sequences of a batch (decode rows) run on the block-streaming decode kernel,
// and the sequences of several query tokens (prefill chunks) on the tcgen05
// chunk kernel.  Otherwise a chunk kernel (tcgen05, or mma.sync for other head
// dims) takes the sequences whose query rows need more than one 16-row tile,
// and the tile-streaming decode kernel the rest.
#include <algorithm>

#include "pk_internal.h"

namespace pk {
namespace {

constexpr size_t kHeaderBytes = 256;     // one scheduler header per kernel

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: decode header | chunk header | split-K counters | merge plan |
// partial log2-sum-exp | partial O.  The headers and the counter region have
// the same offsets and sizes for every pool and batch (the counters are sized
// for kMaxTcKvHeads), so the zeros that every completed call leaves there stay
// valid for the next call, whatever its pool or batch: a workspace, or the
// no-allocation entry point's shared array, can move between pools.  Everything
// after the counters is written before it is read.
constexpr size_t kCountersOff = 2 * kHeaderBytes;
constexpr size_t kZeroedBytes =
    (kCountersOff + (size_t)kMaxSeqsPerLaunch * kMaxTcKvHeads * sizeof(int) + 255) / 256 * 256;

struct Layout {
    size_t hdr_decode, hdr_chunk, counters, merge_plan, partial_lse, partial_o, total;
    int cap_rows;
};

Layout layout(const pk_pool *p, int num_seqs, int n_q_heads) {
    Layout L{};
    const int Hkv = p->n_kv_heads, D = p->head_dim;
    const int g = std::max(1, n_q_heads / Hkv);
    // split items: at most Hkv per sequence plus the ~items_per_cta per CTA that
    // split-K adds; a decode item has g partial rows (the planner coarsens the
    // partitions when a batch of short chunks needs more)
    // (the block-streaming kernel: chunks x heads per stage, rows of g each)
    const long long per_cta =
        std::max((long long)p->tc_ctas * decode_items_per_cta(),
                 p->blk_ok ? (long long)p->sm_count * decode_blocks_chunks_per_cta() * p->blk_hs : 0LL);
    const long long items = (long long)Hkv * std::min(num_seqs, kMaxSeqsPerLaunch) + per_cta;
    L.cap_rows = (int)std::min<long long>(items * std::min(g, kTile), 1LL << 30);
    L.hdr_decode = 0;
    L.hdr_chunk = kHeaderBytes;
    L.counters = kCountersOff;
    size_t off = kZeroedBytes;
    L.merge_plan = off;  // a count, then an int4 per split (sequence, head group)
    off = align_up(off + (size_t)(4 + 4 * kMaxSeqsPerLaunch * Hkv) * sizeof(int), 256);
    L.partial_lse = off;
    off = align_up(off + (size_t)L.cap_rows * sizeof(float), 256);
    L.partial_o = off;
    off = align_up(off + (size_t)L.cap_rows * D * sizeof(float), 256);
    L.total = off;
    return L;
}

}  // namespace

size_t tc_workspace_bytes(const pk_pool *p, int num_seqs, int num_tokens, int n_q_heads,
                          int /*max_blocks_per_seq*/) {
    (void)num_tokens;
    return layout(p, num_seqs, n_q_heads).total;
}

size_t tc_workspace_zeroed_bytes() { return kZeroedBytes; }

int tc_prepare_pool(pk_pool *p) {
    int rc = decode_prepare_pool(p);
    if (rc == PK_OK) rc = decode_blocks_prepare_pool(p);
    if (rc == PK_OK) rc = chunk_prepare_pool(p);
    if (rc == PK_OK) rc = chunk_umma_prepare_pool(p);
    return rc;
}

int launch_attention_tc(const pk_pool *p, const AttnArgs &a, cudaStream_t st) {
    const Layout L = layout(p, a.num_seqs, a.n_q_heads);
    if (a.workspace_bytes < L.total || a.workspace == nullptr)
        return fail(PK_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", a.workspace_bytes, L.total);
    if (((uintptr_t)a.workspace & 255) != 0)
        return fail(PK_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    uint8_t *ws = (uint8_t *)a.workspace;
    DecodeWs w;
    w.header = ws + L.hdr_decode;
    w.counters = (int *)(ws + L.counters);
    w.merge_plan = (int *)(ws + L.merge_plan);
    w.partial_lse = (float *)(ws + L.partial_lse);
    w.partial_o = (float *)(ws + L.partial_o);
    w.cap_rows = L.cap_rows;
    const int g = a.n_q_heads / p->n_kv_heads;
    const bool has_multi = a.num_tokens > a.num_seqs;  // some sequence has several query tokens
    const bool blocks = decode_blocks_applies(p, a);
    // With an append (a.k_new), the block-streaming kernel of a decode-only
    // batch stores the query rows' K/V itself, each just before its block is
    // loaded.  The other paths run the position append kernel first.
    if (!has_multi && blocks) return launch_decode_blocks(p, a, w, false, false, st);
    if (blocks && chunk_umma_applies(p, a)) {
        // a mixed continuous-batching step: the tcgen05 kernel takes every
        // sequence of several query tokens, then the one-token rows stream
        // whole blocks (block-streaming kernel and its merge kernel).  The
        // chunk kernel's CTAs finish unevenly (its items differ in work); the
        // decode kernel, launched behind it, starts its CTAs on the SMs they
        // free and waits for the chunk grid only before it exits.
        int rc = PK_OK;
        if (a.k_new != nullptr) rc = launch_kv_append_at_positions(p, a, st);
        if (rc == PK_OK) rc = launch_chunk_umma(p, a, true, st);
        if (rc == PK_OK) {
            AttnArgs d = a;
            d.k_new = d.v_new = nullptr;  // stored above
            rc = launch_decode_blocks(p, d, w, true, true, st);
        }
        return rc;
    }
    if (a.k_new != nullptr) {
        const int rc = launch_kv_append_at_positions(p, a, st);
        if (rc != PK_OK) return rc;
    }
    // otherwise: sequences whose rows (q_b tokens x g heads) exceed one 16-row
    // tile on a chunk kernel, the rest on the tile-streaming decode kernel
    if (has_multi || g > kTile) {
        const int rc = chunk_umma_applies(p, a) ? launch_chunk_umma(p, a, false, st)
                                                : launch_chunk(p, a, ws + L.hdr_chunk, st);
        if (rc != PK_OK) return rc;
    }
    return launch_decode(p, a, w, st);
}

}  // namespace pk
