// Paged decode attention for bf16 pools (head_dim 64/128/256) for the
// sequences of a batch that have exactly one query token, when a kv head
// serves at most 8 q heads: the decode rows of a continuous-batching step.  In
// a batch that also holds prefill chunks (several query tokens), those
// sequences are left to the chunk kernel, launched on the same stream after
// this kernel.
//
// What is computed ["PagedAttention & Continuous Batching" (study notes),
// "Block tables"; "Batching and PagedAttention", "PagedAttention" item 4]:
// for the query token of sequence b (position c_b - 1) and q head h, softmax
// attention over keys 0..c_b - 1 of kv head h / g, key j read from physical
// block table_b[j / bs] at slot j % bs.
//
// Structure.  Decode attention reads each cached K and V byte once and does
// four flops per byte: it is bound by HBM.  A pool block holds the K (or V)
// rows of all kv heads contiguously ([block][kv head][slot][d]), so a block
// of HS heads is one run of HS * bs rows.  The kernel streams whole blocks:
//   - one producer warp per CTA walks its chunk of the work, looks the blocks up in
//     the block tables and loads each block's K and V rows for HS heads with
//     one TMA box each (all 64-column panels, 128-byte swizzle) into a ring of NS shared-memory
//     stages, a stage being NBS blocks (ST = NBS * bs tokens, up to 64 KiB);
//     a few large copies per block keep HBM busy from one issuing warp;
//   - eight consumer warps own one kv head each (or, for HS < 8, one of
//     8 / HS phases of a head, taking every (8 / HS)-th 16-token tile of a
//     stage).  Per tile: S^T = K Q^T (16 tokens x the head's <= 8 q heads) and
//     O^T += V^T P^T on mma.sync m16n8k16 (bf16 in, fp32 accumulate), with P^T
//     moved into operand order by movmatrix, and an online softmax in fp32.
// Work split (flash-decoding-style split-K, balanced like stream-K): the
// stages of all (sequence, head group) pairs are concatenated and cut into one
// equal chunk per CTA.  The part of a pair inside one chunk is a partition; a
// pair cut into several partitions writes (normalised O, log2-sum-exp) rows per
// partition and kv head, and a merge kernel, launched behind this one as a
// programmatic dependent, combines them once the streaming is over.  (Merging
// inside this kernel, by the last writer of each head, was slower: at the end
// of a launch the other SMs still stream, and a merge's loads wait behind
// their traffic for several microseconds.)  A chunk holds at most two split
// partitions (its first and its last pair), so fewer pairs than chunks are
// split.
//
// Every wait is bounded (2 s); on expiry the kernel records PK_ERR_TIMEOUT,
// waits (bounded) for its own copies in flight and returns.  Block ids are
// range-checked before use.
#include "tc_common.cuh"

#include <algorithm>

namespace pk {
namespace {

using namespace tc;

constexpr int kNC = 8;                        // consumer warps
constexpr int kBlkThreads = (kNC + 1) * 32;   // + one producer warp
constexpr int kStageCap = 64 * 1024;          // K + V bytes of one stage
constexpr int kMinChunkStages = 2;            // smallest chunk
constexpr int kItemSlots = 2;                 // items staged ahead (Q rows + descriptor each)
constexpr float kRescaleLog2 = 8.f;           // lazy softmax rescale threshold (log2 units)
constexpr int kMergeListHead = 4;             // merge kernel's list: count, pad, then int4 entries

enum : int { kFirst = 1, kLast = 2, kEnd = 4 };

// Chunks of the concatenated stages: nb chunks of cb stages (the last one
// shorter), at most one per CTA.
struct ChunkPlan {
    int cb, nb, total;
    __device__ int of(int g) const { return g / cb; }  // chunk holding stage g
    __device__ int begin(int k) const { return k * cb; }
    __device__ int end(int k) const { return min(total, (k + 1) * cb); }
    __device__ int count() const { return nb; }
    // partitions of the stages [start, start + n)
    __device__ int parts(int start, int n) const { return of(start + n - 1) - of(start) + 1; }
};

__device__ inline ChunkPlan make_chunk_plan(int total, int ncta, int scale) {
    ChunkPlan c;
    c.total = total;
    c.cb = max(kMinChunkStages, (int)(((long long)total + ncta - 1) / ncta)) * scale;
    c.nb = (total + c.cb - 1) / c.cb;
    return c;
}

struct StageInfo {
    int slot, st, flags, pad;
};
struct ItemDesc {
    int b, hg, c, qs0, nparts, part, prow, pad;
};

struct BlkParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables, *ctx, *qsl;
    int seq0, nseq, max_blocks, n_q_heads, n_kv_heads, group, block_size, num_blocks, num_tokens;
    int skip_chunks;  // 1: sequences of several query tokens belong to the chunk kernel (skipped)
    // 1: launched behind the chunk kernel of a mixed step, which signals its
    // dependents only once its own wait has returned (the step's rows and the
    // previous call are complete by then).  This grid then reads and writes
    // without a wait of its own, so its CTAs work on the SMs the chunk kernel
    // frees, and waits for the chunk grid only before it exits: the grids
    // after it on the stream still find both finished.
    int behind_chunk;
    int HS, NBS, ST, NPH, NS;  // geometry: heads / blocks / tokens per stage, phases, stages
    int ncta, cap_rows;
    float scale_log2;
    int *mplan;                      // the merge kernel's list of split pairs
    // the decode rows' own K/V ([num_tokens, n_kv_heads, D]) to store at their
    // positions before their blocks are read, and the pool they go to (a
    // decode-only batch); k_new == nullptr: nothing to store
    const __nv_bfloat16 *k_new, *v_new;
    __nv_bfloat16 *kpool, *vpool;
    float *partial_o, *partial_lse;  // [row][D], [row]
    int *err;
    // shared-memory layout (byte offsets from the 1024-aligned base)
    uint32_t stage_bytes, qslot_bytes, off_q, off_scr, off_plan, off_desc, off_info, off_bar, total;
};

// Shared-memory layout of one launch.
template <int D>
void blk_layout(BlkParams &p) {
    constexpr int KS = D / 16;
    auto up = [](uint32_t x, uint32_t a) { return (x + a - 1) / a * a; };
    p.stage_bytes = (uint32_t)p.NBS * p.HS * p.block_size * D * 4;
    p.qslot_bytes = up((uint32_t)p.HS * p.group * D * 2, 128);
    uint32_t off = (uint32_t)p.NS * p.stage_bytes;
    p.off_q = off;
    off += kItemSlots * p.qslot_bytes;
    p.off_scr = off;
    if (p.NPH > 1) off += (uint32_t)(kNC - p.HS) * 32 * (KS * 4 + 4) * 4;
    p.off_plan = off;
    off += up(4 * kPlanLen * 4, 16);
    p.off_desc = off;
    off += kItemSlots * sizeof(ItemDesc);
    p.off_info = off;
    off += (uint32_t)p.NS * sizeof(StageInfo);
    p.off_bar = up(off, 8);
    off = p.off_bar + (uint32_t)(2 * p.NS + 2 * kItemSlots + 1) * 8;
    p.total = off + 1024;  // + alignment slack
}

template <int D>
__global__ void __launch_bounds__(kBlkThreads, 1)
attention_decode_blocks_kernel(const __grid_constant__ CUtensorMap tmk,
                               const __grid_constant__ CUtensorMap tmv, const BlkParams prm) {
    constexpr int KS = D / 16;
    constexpr int NPN = D / 64;  // 64-column panels
    extern __shared__ uint8_t smem_raw[];
    // Launched as a programmatic dependent of the previous kernel on the stream
    // (the KV append or block copy, which write pool rows only).  The plan, the
    // query rows and the block tables are read while that kernel may still
    // run; the pool is read, and anything written, only after
    // griddepcontrol.wait: by the producer before its first K/V copy, by the
    // consumers at their start.
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NS = prm.NS, HS = prm.HS, NBS = prm.NBS, ST = prm.ST, NPH = prm.NPH;
    const int g = prm.group, Hq = prm.n_q_heads, Hkv = prm.n_kv_heads, bs = prm.block_size;
    const int NHG = Hkv / HS, nseq = prm.nseq;
    const int PR = HS * bs;                                  // rows of a block's head group
    const uint32_t panel_bytes = (uint32_t)PR * 128;         // one 64-column panel of a block
    const uint32_t piece_bytes = panel_bytes * NPN;          // a block's K (or V) rows
    int *stage_pre = (int *)(sm + prm.off_plan);  // stages of sequences 0..i-1 (all head groups)
    int *prow_pre = stage_pre + kPlanLen;         // split-K partial rows of sequences 0..i-1
    int *s_qsl = prow_pre + kPlanLen;
    int *s_ctx = s_qsl + kPlanLen;
    ItemDesc *descs = (ItemDesc *)(sm + prm.off_desc);
    StageInfo *infos = (StageInfo *)(sm + prm.off_info);
    uint64_t *full = (uint64_t *)(sm + prm.off_bar);
    uint64_t *empty = full + NS;
    uint64_t *qfull = empty + NS;
    uint64_t *iempty = qfull + kItemSlots;
    uint64_t *cbar = iempty + kItemSlots;  // barrier of the consumer warps
    __shared__ ChunkPlan s_cp;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kNC);
        }
        for (int s = 0; s < kItemSlots; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&iempty[s], kNC);
        }
        mbar_init(cbar, kNC);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the window's query offsets and context lengths, one load per thread
    for (int i = threadIdx.x; i <= nseq; i += kBlkThreads) {
        s_qsl[i] = __ldg(prm.qsl + prm.seq0 + i);
        if (i < nseq) s_ctx[i] = __ldg(prm.ctx + prm.seq0 + i);
    }
    __syncthreads();
    // ---------------------------------------------------------------- plan
    // per sequence: S_b = ceil(c_b / ST) stages per head group; chunk size CS;
    // a (sequence, head group) spanning several chunks has one partition per
    // chunk, each with HS * g partial rows
    if (warp == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        int run = 0;
        for (int base = 0; base < nseq; base += 32) {
            const int i = base + lane;
            int ns = 0;
            if (i < nseq) {
                const int s0 = s_qsl[i], s1 = s_qsl[i + 1], c = s_ctx[i];
                const bool ok = s0 >= 0 && s1 <= prm.num_tokens && s1 - s0 >= 1 && c >= s1 - s0 &&
                                (long long)(c + bs - 1) / bs <= prm.max_blocks &&
                                (s1 - s0 == 1 || prm.skip_chunks);
                if (!ok) record_error(prm.err, PK_ERR_BAD_INDEX);
                else if (s1 - s0 == 1) ns = NHG * ((c + ST - 1) / ST);
            }
            int inc = ns;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            if (i < nseq) stage_pre[i + 1] = run + inc;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) stage_pre[0] = 0;
        __syncwarp();
        const int total = run;
        ChunkPlan cp = make_chunk_plan(total, prm.ncta, 1);
        for (int attempt = 0; attempt < 8; ++attempt) {
            int runp = 0;
            for (int base = 0; base < nseq; base += 32) {
                const int i = base + lane;
                int np = 0;
                if (i < nseq) {
                    const int sb = (stage_pre[i + 1] - stage_pre[i]) / NHG;
                    for (int hg = 0; hg < NHG && sb > 0; ++hg) {
                        const int n = cp.parts(stage_pre[i] + hg * sb, sb);
                        if (n > 1) np += n * HS * g;
                    }
                }
                int inc = np;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += y;
                }
                if (i < nseq) prow_pre[i + 1] = runp + inc;
                runp += __shfl_sync(0xffffffffu, inc, 31);
            }
            if (runp <= prm.cap_rows) break;
            // more partial rows than the workspace holds: coarser chunks, finally
            // one chunk for everything (no split)
            if (attempt < 6) {
                cp = make_chunk_plan(total, prm.ncta, 2 << attempt);
            } else {
                cp.cb = max(total, 1);
                cp.nb = total > 0 ? 1 : 0;
            }
        }
        if (lane == 0) {
            prow_pre[0] = 0;
            s_cp = cp;
        }
        __syncwarp();
    }
    // a merge kernel, if one follows, may be scheduled now; it waits for this grid to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    const ChunkPlan cp = s_cp;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        // CTA i takes chunk i
        const int nchunks = cp.count();
        int pending = (int)blockIdx.x;
        int n_stage = 0, n_item = 0;
        bool waited = prm.behind_chunk != 0;  // griddepcontrol.wait done (or not needed)
        const uint64_t stream_pol = l2_evict_first_policy();  // K/V rows are read once
        auto chunk_entry = [&](int b, int blk_base) -> int {
            const int nblk = (s_ctx[b] + bs - 1) / bs;
            const int e = blk_base + lane;
            return e < nblk ? __ldg(prm.tables + (long long)(prm.seq0 + b) * prm.max_blocks + e) : 0;
        };
        // the token of sequence b's (one) query row
        auto d_tok = [&](int b) -> int { return s_qsl[b]; };
        // query token tok's K and V rows of kv heads h0 .. h0 + nh - 1 into block
        // phys at offset off (16-byte vectors over the warp's lanes)
        auto store_row = [&](int tok, int phys, int off, int h0, int nh) {
            constexpr int RC = D / 8;  // 16-byte chunks of a row
            const uint4 *ks = (const uint4 *)prm.k_new, *vs = (const uint4 *)prm.v_new;
            uint4 *kd = (uint4 *)prm.kpool, *vd = (uint4 *)prm.vpool;
            for (int i = lane; i < nh * RC; i += 32) {
                const int h = h0 + i / RC, e = i % RC;
                const long long src = ((long long)tok * Hkv + h) * RC + e;
                const long long dst = (((long long)phys * Hkv + h) * bs + off) * RC + e;
                kd[dst] = __ldg(ks + src);
                vd[dst] = __ldg(vs + src);
            }
        };
        // Items (partitions) in chunk order.  The next item is found, and its
        // first two table chunks requested, while the current one's stages
        // are issued, so the table lookups of an item start without a wait.
        struct PItem {
            int b, hg, st0, cnt, nparts, part, prow, tab0, tab1;
        };
        int g0 = 0, g1 = 0;
        auto next_item = [&](PItem &it) -> bool {
            while (g0 >= g1) {
                const int chunk = pending;
                if (chunk >= nchunks) return false;
                pending = nchunks;  // one chunk per CTA
                g0 = cp.begin(chunk);
                g1 = cp.end(chunk);
            }
            // the partition of one (sequence, head group) inside the chunk
            const int b = find_seq(stage_pre, nseq, g0);
            const int sb = (stage_pre[b + 1] - stage_pre[b]) / NHG;
            const int local = g0 - stage_pre[b];
            it.b = b;
            it.hg = local / sb;
            it.st0 = local - it.hg * sb;
            it.cnt = min(sb - it.st0, g1 - g0);
            const int start = stage_pre[b] + it.hg * sb;
            it.nparts = cp.parts(start, sb);
            it.part = cp.of(g0) - cp.of(start);
            it.prow = prow_pre[b];
            for (int h = 0; h < it.hg; ++h) {
                const int n = cp.parts(stage_pre[b] + h * sb, sb);
                if (n > 1) it.prow += n * HS * g;
            }
            const int base = (it.st0 * NBS) & ~31;
            it.tab0 = chunk_entry(b, base);
            it.tab1 = chunk_entry(b, base + 32);
            g0 += it.cnt;
            return true;
        };
        PItem cur, nxt;
        bool have = next_item(cur);
        while (ok && have) {
            const bool have_next = next_item(nxt);
            const int b = cur.b, hg = cur.hg, c = s_ctx[b];
            const int slot = n_item % kItemSlots;
            if (n_item >= kItemSlots &&
                !mbar_wait(&iempty[slot], (uint32_t)(n_item / kItemSlots - 1) & 1)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                ItemDesc &d = descs[slot];
                d.b = b;
                d.hg = hg;
                d.c = c;
                d.qs0 = s_qsl[b];
                d.nparts = cur.nparts;
                d.part = cur.part;
                d.prow = cur.prow;
                const uint32_t qb = (uint32_t)HS * g * D * 2;
                mbar_arrive_expect_tx(&qfull[slot], qb);
                bulk_load(sm + prm.off_q + slot * prm.qslot_bytes,
                          prm.q + ((long long)s_qsl[b] * Hq + hg * HS * g) * D, qb, &qfull[slot]);
            }
            __syncwarp();
            ++n_item;
            // block table lookups: this lane holds entry cur_base + lane; the
            // following 32 entries are in flight
            int cur_base = (cur.st0 * NBS) & ~31, cur_tab = cur.tab0, nxt_tab = cur.tab1;
            // the table entry of block blk (non-decreasing over the item); a bad id
            // is recorded and comes back as -1
            auto table_get = [&](int blk) -> int {
                while (blk >= cur_base + 32) {
                    cur_base += 32;
                    cur_tab = nxt_tab;
                    nxt_tab = chunk_entry(b, cur_base + 32);
                }
                const int phys = __shfl_sync(0xffffffffu, cur_tab, blk - cur_base);
                if (phys < 0 || phys >= prm.num_blocks) {
                    if (lane == 0) record_error(prm.err, PK_ERR_BAD_INDEX);
                    return -1;
                }
                return phys;
            };
            const int nblk = (c + bs - 1) / bs;
            // with an append, the row's own K/V go to position c - 1 (block
            // new_blk, offset new_off) before that block is loaded
            const int new_blk = prm.k_new != nullptr ? (c - 1) / bs : -1;
            const int new_off = (c - 1) - new_blk * bs;
            if (!waited) {  // the preceding kernel's pool rows are visible from here on
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
            }
            // when this item reaches the new row's block, that row's K/V (heads of
            // this group, contiguous in k_new) are loaded now and stored there
            constexpr int RCd = D / 8, UP = 4;
            const int nrow = HS * RCd;
            const bool pre = new_blk >= 0 && new_blk / NBS >= cur.st0 && new_blk / NBS < cur.st0 + cur.cnt &&
                             nrow <= 32 * UP;
            uint4 pk[UP], pv[UP];
            if (pre) {
                const long long src0 = ((long long)d_tok(b) * Hkv + hg * HS) * RCd;
#pragma unroll
                for (int u = 0; u < UP; ++u) {
                    const int i = u * 32 + lane;
                    if (i < nrow) {
                        pk[u] = __ldg((const uint4 *)prm.k_new + src0 + i);
                        pv[u] = __ldg((const uint4 *)prm.v_new + src0 + i);
                    }
                }
            }
            for (int st = cur.st0; st < cur.st0 + cur.cnt; ++st) {
                const int s = n_stage % NS;
                if (n_stage >= NS && !mbar_wait(&empty[s], ((n_stage / NS) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int blk0 = st * NBS;
                const int np = min(NBS, nblk - blk0);  // blocks of this stage inside the context
                if (lane == 0) {
                    StageInfo &inf = infos[s];
                    inf.slot = slot;
                    inf.st = st;
                    inf.flags = (st == cur.st0 ? kFirst : 0) | (st == cur.st0 + cur.cnt - 1 ? kLast : 0);
                    mbar_arrive_expect_tx(&full[s], (uint32_t)np * piece_bytes * 2);
                }
                uint8_t *kst = sm + (size_t)s * prm.stage_bytes;
                uint8_t *vst = kst + (size_t)NBS * piece_bytes;
                for (int j = 0; j < np; ++j) {
                    const int raw = table_get(blk0 + j);
                    const int phys = raw < 0 ? 0 : raw;
                    if (blk0 + j == new_blk) {
                        if (raw >= 0 && pre) {
                            uint4 *kd = (uint4 *)prm.kpool, *vd = (uint4 *)prm.vpool;
#pragma unroll
                            for (int u = 0; u < UP; ++u) {
                                const int i = u * 32 + lane;
                                if (i < nrow) {
                                    const long long dst =
                                        (((long long)raw * Hkv + hg * HS + i / RCd) * bs + new_off) * RCd + i % RCd;
                                    kd[dst] = pk[u];
                                    vd[dst] = pv[u];
                                }
                            }
                        } else if (raw >= 0) {
                            store_row(d_tok(b), raw, new_off, hg * HS, HS);
                        }
                        // the generic-proxy stores before the TMA box that reads them
                        asm volatile("fence.proxy.async.global;" ::: "memory");
                        __syncwarp();
                    }
                    const int y = (phys * Hkv + hg * HS) * bs;
                    if (lane == 0) {  // all panels of the block's rows: one box for K, one for V
                        tma_load_3d_hint(kst + j * piece_bytes, &tmk, 0, y, 0, &full[s], stream_pol);
                        tma_load_3d_hint(vst + j * piece_bytes, &tmv, 0, y, 0, &full[s], stream_pol);
                    }
                }
                __syncwarp();
                ++n_stage;
            }
            cur = nxt;
            have = have_next;
        }
        if (ok) {
            // end marker
            const int s = n_stage % NS;
            if (n_stage >= NS && !mbar_wait(&empty[s], ((n_stage / NS) - 1) & 1)) ok = false;
            if (ok) {
                if (lane == 0) {
                    infos[s].flags = kEnd;
                    mbar_arrive(&full[s]);
                }
                ++n_stage;
            }
        }
        if (blockIdx.x == 0) {
            // the merge kernel's work list: (sequence, head group, first partial
            // row, partitions) of every pair cut into several partitions.  The
            // previous merge kernel on the stream reads its list until its grid
            // ends, so this one is written after the wait.
            if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");
            int n_split = 0;
            for (int base = 0; base < nseq; base += 32) {
                const int i = base + lane;
                const int sb = i < nseq ? (stage_pre[i + 1] - stage_pre[i]) / NHG : 0;
                int prow = i < nseq ? prow_pre[i] : 0;
                for (int hg = 0; hg < NHG; ++hg) {
                    const int n = sb > 0 ? cp.parts(stage_pre[i] + hg * sb, sb) : 1;
                    const unsigned m = __ballot_sync(0xffffffffu, n > 1);
                    if (n > 1) {
                        int4 *e = (int4 *)(prm.mplan + kMergeListHead) + n_split + __popc(m & ((1u << lane) - 1));
                        *e = make_int4(i, hg, prow, n);
                        prow += n * HS * g;
                    }
                    n_split += __popc(m);
                }
            }
            if (lane == 0) prm.mplan[0] = n_split;
        }
        if (!ok) {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            // never leave with a copy still writing into this CTA's shared memory
            for (int n = max(0, n_stage - NS); n < n_stage; ++n)
                mbar_wait(&full[n % NS], (uint32_t)(n / NS) & 1);
            for (int k = max(0, n_item - kItemSlots); k < n_item; ++k)
                mbar_wait(&qfull[k % kItemSlots], (uint32_t)(k / kItemSlots) & 1);
        }
    } else {
        // ---------------------------------------------------------- consumers
        if (!prm.behind_chunk) asm volatile("griddepcontrol.wait;" ::: "memory");  // before any write
        const int cw = warp - 1, hl = cw % HS, ph = cw / HS;
        const int qr = lane >> 2, qc = (lane & 3) * 2;
        const int mi = lane >> 3, rr = lane & 7;
        const int a_row = (mi & 1) * 8 + rr, a_col = (mi >> 1) * 8;  // K rows (A of S^T)
        const int v_row = (mi >> 1) * 8 + rr, v_col = (mi & 1) * 8;  // V rows (A of O^T, transposed)
        uint32_t qb[KS][2];
        float ot[KS][4];
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads qc, qc + 1
        int c = 0;
        uint32_t qph = 0, cph = 0;
        // all consumer warps meet (bounded: false after the wait limit)
        auto consumer_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(cbar);
            const bool r = mbar_wait(cbar, cph);
            cph ^= 1u;
            return r;
        };
        // byte offset of stage-relative token tau's row (head hl) in a K or V part, and its swizzle phase
        auto row_of = [&](int tau, uint32_t &off, int &sw) {
            const int pc = tau / bs, t = tau - pc * bs;
            const int r = hl * bs + t;
            off = (uint32_t)pc * piece_bytes + (uint32_t)r * 128;
            sw = r & 7;
        };
        auto begin_item = [&](int slot) -> bool {
            if (!mbar_wait(&qfull[slot], (qph >> slot) & 1)) return false;
            qph ^= 1u << slot;
            c = descs[slot].c;
            const uint8_t *qh = sm + prm.off_q + slot * prm.qslot_bytes + (size_t)(hl * g + qr) * D * 2;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int col = (kk * 16 + qc) * 2;
                qb[kk][0] = qr < g ? *(const uint32_t *)(qh + col) : 0u;
                qb[kk][1] = qr < g ? *(const uint32_t *)(qh + col + 16) : 0u;
            }
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
            return true;
        };
        // one 16-token tile (stage-relative tokens tau0..tau0+15, sequence tokens tok0..)
        auto tile = [&](uint8_t *kst, uint8_t *vst, int tau0, int tok0) {
            const int valid = c - tok0;
            if (valid < kTile) {
                // tail: clear V rows past the context (stale or never-written slots)
                for (int ch = lane; ch < (kTile - valid) * (D / 8); ch += 32) {
                    const int row = valid + ch / (D / 8), col = (ch % (D / 8)) * 8;
                    uint32_t off;
                    int sw;
                    row_of(tau0 + row, off, sw);
                    *(uint4 *)(vst + off + (col >> 6) * panel_bytes + ((((col & 63) >> 3) ^ sw) << 4)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async();  // the stage is rewritten by TMA later
                __syncwarp();
            }
            uint32_t koff, voff;
            int ksw, vsw;
            row_of(tau0 + a_row, koff, ksw);
            row_of(tau0 + v_row, voff, vsw);
            const uint32_t ka = smem_u32(kst) + koff, va = smem_u32(vst) + voff;
            float sa[4][4] = {};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int col = kk * 16 + a_col;
                uint32_t a0, a1, a2, a3;
                ldsm_x4(ka + (col >> 6) * panel_bytes + ((((col & 63) >> 3) ^ ksw) << 4), a0, a1, a2, a3);
                mma_bf16(sa[kk & 3], a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            }
            // four accumulator chains; s0, s1: token qr, heads qc, qc + 1; s2, s3: token qr + 8
            auto sum4 = [&](int i) { return ((sa[0][i] + sa[1][i]) + (sa[2][i] + sa[3][i])) * prm.scale_log2; };
            float s0 = sum4(0), s1 = sum4(1), s2 = sum4(2), s3 = sum4(3);
            if (qr >= valid) s0 = s1 = -INFINITY;
            if (qr + 8 >= valid) s2 = s3 = -INFINITY;
            // Lazy rescaling: the running reference m moves (and O, l are
            // rescaled) only when a score exceeds it by more than kRescaleLog2,
            // so 2^(s - m) stays below 2^kRescaleLog2 (exact in the end: o = O / l
            // and lse = m + log2 l hold for any reference).  The vote keeps the
            // branch warp-uniform.
            const float la = fmaxf(s0, s2), lb = fmaxf(s1, s3);
            if (__any_sync(0xffffffffu, la > m0 + kRescaleLog2 || lb > m1 + kRescaleLog2)) {
                float ma = la, mb = lb;
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) {
                    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, x));
                    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, x));
                }
                const float na = fmaxf(m0, ma), nb = fmaxf(m1, mb);
                const float ala = na == -INFINITY ? 1.f : fast_exp2(m0 - na);
                const float alb = nb == -INFINITY ? 1.f : fast_exp2(m1 - nb);
                m0 = na;
                m1 = nb;
                l0 *= ala;
                l1 *= alb;
#pragma unroll
                for (int mt = 0; mt < KS; ++mt) {
                    ot[mt][0] *= ala;
                    ot[mt][1] *= alb;
                    ot[mt][2] *= ala;
                    ot[mt][3] *= alb;
                }
            }
            const float ba = m0 == -INFINITY ? 0.f : m0, bb = m1 == -INFINITY ? 0.f : m1;
            const float p0 = fast_exp2(s0 - ba), p1 = fast_exp2(s1 - bb);
            const float p2 = fast_exp2(s2 - ba), p3 = fast_exp2(s3 - bb);
            l0 += p0 + p2;
            l1 += p1 + p3;
            // P^T as the B fragment: transpose the two 8x8 (token x head) blocks
            const uint32_t b0 = movmatrix_trans(pack_bf16(p0, p1));
            const uint32_t b1 = movmatrix_trans(pack_bf16(p2, p3));
            // O^T (16 d-rows x 8 heads per m-tile) += V^T P^T
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const int col = mt * 16 + v_col;
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(va + (col >> 6) * panel_bytes + ((((col & 63) >> 3) ^ vsw) << 4), a0, a1, a2, a3);
                mma_bf16(ot[mt], a0, a1, a2, a3, b0, b1);
            }
        };
        float *scr = (float *)(sm + prm.off_scr);
        constexpr int kScr = KS * 4 + 4;  // floats per lane of one warp's state
        auto finish_item = [&](int slot) -> bool {
            const ItemDesc d = descs[slot];
            if (NPH > 1) {
                // phases of one head: fold phases 1.. into phase 0 through shared memory
                if (ph > 0) {
                    float *w = scr + (size_t)(cw - HS) * 32 * kScr;
#pragma unroll
                    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) w[(mt * 4 + i) * 32 + lane] = ot[mt][i];
                    w[(KS * 4 + 0) * 32 + lane] = m0;
                    w[(KS * 4 + 1) * 32 + lane] = m1;
                    w[(KS * 4 + 2) * 32 + lane] = l0;
                    w[(KS * 4 + 3) * 32 + lane] = l1;
                }
                if (!consumer_sync()) return false;
                if (ph == 0) {
                    for (int q = 1; q < NPH; ++q) {
                        const float *w = scr + (size_t)(hl + q * HS - HS) * 32 * kScr;
                        const float xm0 = w[(KS * 4 + 0) * 32 + lane], xm1 = w[(KS * 4 + 1) * 32 + lane];
                        const float xl0 = w[(KS * 4 + 2) * 32 + lane], xl1 = w[(KS * 4 + 3) * 32 + lane];
                        const float n0 = fmaxf(m0, xm0), n1 = fmaxf(m1, xm1);
                        const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
                        const float a0 = fast_exp2(m0 - b0), x0 = fast_exp2(xm0 - b0);
                        const float a1 = fast_exp2(m1 - b1), x1 = fast_exp2(xm1 - b1);
                        l0 = l0 * a0 + xl0 * x0;
                        l1 = l1 * a1 + xl1 * x1;
                        m0 = n0;
                        m1 = n1;
#pragma unroll
                        for (int mt = 0; mt < KS; ++mt) {
                            ot[mt][0] = ot[mt][0] * a0 + w[(mt * 4 + 0) * 32 + lane] * x0;
                            ot[mt][1] = ot[mt][1] * a1 + w[(mt * 4 + 1) * 32 + lane] * x1;
                            ot[mt][2] = ot[mt][2] * a0 + w[(mt * 4 + 2) * 32 + lane] * x0;
                            ot[mt][3] = ot[mt][3] * a1 + w[(mt * 4 + 3) * 32 + lane] * x1;
                        }
                    }
                }
                if (!consumer_sync()) return false;  // the scratch is free again
            }
            const bool split = d.nparts > 1;
            if (ph == 0) {
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) {  // sums over the token lanes of each head
                    l0 += __shfl_xor_sync(0xffffffffu, l0, x);
                    l1 += __shfl_xor_sync(0xffffffffu, l1, x);
                }
                const float ia = l0 > 0.f ? 1.f / l0 : 0.f, ib = l1 > 0.f ? 1.f / l1 : 0.f;
                const int ha = qc, hb = qc + 1;  // heads of this lane's accumulators
                const bool va_ = ha < g, vb_ = hb < g;
                const int kvh = d.hg * HS + hl;
                if (!split) {
                    __nv_bfloat16 *oa = prm.out + ((long long)d.qs0 * Hq + kvh * g + ha) * D;
                    __nv_bfloat16 *ob = oa + D;
#pragma unroll
                    for (int mt = 0; mt < KS; ++mt) {
                        const int d0 = mt * 16 + qr;
                        if (va_) {
                            oa[d0] = __float2bfloat16_rn(ot[mt][0] * ia);
                            oa[d0 + 8] = __float2bfloat16_rn(ot[mt][2] * ia);
                        }
                        if (vb_) {
                            ob[d0] = __float2bfloat16_rn(ot[mt][1] * ib);
                            ob[d0 + 8] = __float2bfloat16_rn(ot[mt][3] * ib);
                        }
                    }
                } else {
                    // partial rows are read back by the merge kernel: kept in L2
                    // past the K/V stream that follows them
                    const uint64_t keep = l2_evict_last_policy();
                    const int row = d.prow + d.part * HS * g + hl * g;
                    float *pa_ = prm.partial_o + (size_t)(row + ha) * D;
                    float *pb_ = pa_ + D;
#pragma unroll
                    for (int mt = 0; mt < KS; ++mt) {
                        const int d0 = mt * 16 + qr;
                        if (va_) {
                            st_l2_keep(pa_ + d0, ot[mt][0] * ia, keep);
                            st_l2_keep(pa_ + d0 + 8, ot[mt][2] * ia, keep);
                        }
                        if (vb_) {
                            st_l2_keep(pb_ + d0, ot[mt][1] * ib, keep);
                            st_l2_keep(pb_ + d0 + 8, ot[mt][3] * ib, keep);
                        }
                    }
                    if (qr == 0) {
                        float *pl = prm.partial_lse + (size_t)row;
                        if (va_) st_l2_keep(pl + ha, l0 > 0.f ? m0 + __log2f(l0) : -INFINITY, keep);
                        if (vb_) st_l2_keep(pl + hb, l1 > 0.f ? m1 + __log2f(l1) : -INFINITY, keep);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&iempty[slot]);
            return true;
        };

        for (int n = 0;; ++n) {
            const int s = n % NS;
            if (!mbar_wait(&full[s], (uint32_t)(n / NS) & 1)) {
                ok = false;
                break;
            }
            const StageInfo inf = infos[s];
            if (inf.flags & kEnd) break;
            if ((inf.flags & kFirst) && !begin_item(inf.slot)) {
                ok = false;
                break;
            }
            uint8_t *kst = sm + (size_t)s * prm.stage_bytes;
            uint8_t *vst = kst + (size_t)NBS * piece_bytes;
            const int tok_stage = inf.st * ST;
            for (int j = ph; j * kTile < ST; j += NPH) {
                const int tok0 = tok_stage + j * kTile;
                if (tok0 >= c) break;
                tile(kst, vst, j * kTile, tok0);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if ((inf.flags & kLast) && !finish_item(inf.slot)) {
                ok = false;
                break;
            }
        }
        if (!ok && lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
    }
    __syncthreads();
    // behind a chunk kernel: the CTA leaves only once the chunk grid has finished
    if (prm.behind_chunk && threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Merge kernel [flash-decoding combination].  For every (sequence, head
// group) that the streaming kernel cut into several partitions, each output
// row (q head hg * HS * g + r of the sequence's token) is
// out = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M), M = max_p lse_p, over
// the partitions' normalised rows o_p and log2-sum-exps lse_p.  Launched as a
// programmatic dependent of the streaming kernel, its CTAs are resident
// before that grid ends and start the moment it does, when the memory system
// is quiet and the partial rows are still in L2.
// The streaming kernel lists the split pairs.  blockIdx.x = list entry,
// blockIdx.y = a block of kMergeThreads outputs (row, 4 columns) of that
// pair; one thread per output folds the partitions eight at a time, all of a
// batch's loads issued before the first is used.  No shared memory, no
// barrier: a block past the list's end returns at once.
struct MergeParams {
    __nv_bfloat16 *out;
    const int32_t *qsl;
    const int *mplan;
    const float *partial_o, *partial_lse;
    int seq0, n_q_heads, group, HS;
};

constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 8;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) attention_merge_kernel(const MergeParams mp) {
    // the next kernel on the stream may start launching (it waits for this
    // grid before touching memory); the streaming kernel has finished once
    // the wait returns
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int HG = mp.HS * mp.group;
    const int unit = blockIdx.y * kMergeThreads + threadIdx.x;
    const int n_split = __ldcg(mp.mplan);
    const int4 e = __ldcg((const int4 *)(mp.mplan + kMergeListHead) + blockIdx.x);
    if ((int)blockIdx.x >= n_split || unit >= HG * (D / 4)) return;
    const int b = e.x, hg = e.y, prow = e.z, nparts = e.w;  // sequence, head group, first row, partitions
    const int r = unit / (D / 4), c4 = unit % (D / 4);
    const float *lse = mp.partial_lse + prow + r;
    const float4 *po = (const float4 *)(mp.partial_o + (size_t)(prow + r) * D) + c4;
    float M = -INFINITY, den = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int q0 = 0; q0 < nparts; q0 += kMergeBatch) {
        float l[kMergeBatch];
        float4 x[kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            l[i] = -INFINITY;
            x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (q0 + i < nparts) {
                l[i] = __ldcg(lse + (size_t)(q0 + i) * HG);
                x[i] = __ldcg(po + (size_t)(q0 + i) * HG * (D / 4));
            }
        }
        float bm = M;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) bm = fmaxf(bm, l[i]);
        if (bm == -INFINITY) continue;
        const float a = M == -INFINITY ? 0.f : fast_exp2(M - bm);
        den *= a;
        acc.x *= a;
        acc.y *= a;
        acc.z *= a;
        acc.w *= a;
        M = bm;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            const float w = l[i] == -INFINITY ? 0.f : fast_exp2(l[i] - M);
            den += w;
            acc.x += w * x[i].x;
            acc.y += w * x[i].y;
            acc.z += w * x[i].z;
            acc.w += w * x[i].w;
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const long long orow = (long long)__ldg(mp.qsl + mp.seq0 + b) * mp.n_q_heads + hg * HG + r;
    uint2 pk;
    pk.x = pack_bf16(acc.x * inv, acc.y * inv);
    pk.y = pack_bf16(acc.z * inv, acc.w * inv);
    *(uint2 *)(mp.out + orow * D + c4 * 4) = pk;
}

// The largest dynamic shared memory a launch may ask for: the device's opt-in
// limit per block less the kernel's static shared memory.
template <int D>
int blocks_prepare(pk_pool *p) {
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
    cudaFuncAttributes fa{};
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, attention_decode_blocks_kernel<D>);
    if (e != cudaSuccess) return cuda_fail(e, "decode (block stream) attributes");
    p->blk_smem_max = optin - (int)fa.sharedSizeBytes;
    e = cudaFuncSetAttribute(attention_decode_blocks_kernel<D>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, p->blk_smem_max);
    if (e != cudaSuccess) return cuda_fail(e, "set decode (block stream) smem size");
    return PK_OK;
}

template <int D>
int blocks_launch(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, bool skip_chunks, bool behind_chunk,
                  cudaStream_t st) {
    BlkParams tp{};
    tp.skip_chunks = skip_chunks ? 1 : 0;
    tp.q = (const __nv_bfloat16 *)a.q;
    tp.out = (__nv_bfloat16 *)a.out;
    tp.tables = a.block_tables;
    tp.ctx = a.context_lens;
    tp.qsl = a.query_start_lens;
    tp.max_blocks = a.max_blocks_per_seq;
    tp.n_q_heads = a.n_q_heads;
    tp.n_kv_heads = p->n_kv_heads;
    tp.group = a.n_q_heads / p->n_kv_heads;
    tp.block_size = p->block_size;
    tp.num_blocks = p->num_blocks;
    tp.num_tokens = a.num_tokens;
    tp.HS = p->blk_hs;
    tp.NBS = p->blk_nbs;
    tp.ST = p->blk_nbs * p->block_size;
    tp.NPH = kNC / p->blk_hs;
    tp.ncta = p->sm_count;
    tp.cap_rows = w.cap_rows;
    tp.scale_log2 = a.scale * 1.4426950408889634f;
    tp.mplan = w.merge_plan;
    tp.k_new = (const __nv_bfloat16 *)a.k_new;
    tp.v_new = (const __nv_bfloat16 *)a.v_new;
    tp.kpool = (__nv_bfloat16 *)p->k_base;
    tp.vpool = (__nv_bfloat16 *)p->v_base;
    tp.partial_o = w.partial_o;
    tp.partial_lse = w.partial_lse;
    tp.err = p->d_err;
    tp.NS = 3;
    blk_layout<D>(tp);
    if (tp.total > (uint32_t)p->blk_smem_max) {
        tp.NS = 2;
        blk_layout<D>(tp);
    }
    if (tp.total > (uint32_t)p->blk_smem_max)
        return fail(PK_ERR_UNSUPPORTED, "decode attention: %u bytes of shared memory", tp.total);
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        tp.seq0 = s0;
        tp.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        tp.behind_chunk = behind_chunk && s0 == 0 ? 1 : 0;  // later windows follow a merge kernel
        {
            cudaLaunchConfig_t c0 = {};
            c0.gridDim = dim3(tp.ncta);
            c0.blockDim = dim3(kBlkThreads);
            c0.dynamicSmemBytes = tp.total;
            c0.stream = st;
            cudaLaunchAttribute a0[1];
            a0[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            a0[0].val.programmaticStreamSerializationAllowed = 1;
            c0.attrs = a0;
            c0.numAttrs = 1;
            const cudaError_t e0 = cudaLaunchKernelEx(&c0, attention_decode_blocks_kernel<D>, p->tmap_kb, p->tmap_vb, tp);
            if (e0 != cudaSuccess) return cuda_fail(e0, "decode attention launch");
        }
        MergeParams mp;
        mp.out = tp.out;
        mp.qsl = tp.qsl;
        mp.mplan = tp.mplan;
        mp.partial_o = tp.partial_o;
        mp.partial_lse = tp.partial_lse;
        mp.seq0 = tp.seq0;
        mp.n_q_heads = tp.n_q_heads;
        mp.group = tp.group;
        mp.HS = tp.HS;
        const int units = tp.HS * tp.group * (D / 4);
        cudaLaunchConfig_t cfg = {};
        // one block row per possible split pair (sequence, head group): each split
        // pair holds a chunk boundary, so there are fewer than the chunks (at most
        // one per SM); blocks past the list's end return at once
        const int pairs = tp.nseq * (tp.n_kv_heads / tp.HS);
        cfg.gridDim = dim3(std::min(pairs, tp.ncta), (units + kMergeThreads - 1) / kMergeThreads);
        cfg.blockDim = dim3(kMergeThreads);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, attention_merge_kernel<D>, mp);
        if (e != cudaSuccess) return cuda_fail(e, "split-K merge launch");
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "decode attention launch");
}

}  // namespace

// Stage geometry of a pool: HS = the largest power of two dividing n_kv_heads
// (at most 8) whose block (K + V of HS heads) fits a stage, halved until a
// stage of whole blocks holds a multiple of 16 tokens; NBS = blocks per stage.
int decode_blocks_prepare_pool(pk_pool *p) {
    p->blk_ok = false;
    const int D = p->head_dim, bs = p->block_size;
    int hs = 1;
    while (hs < 8 && p->n_kv_heads % (hs * 2) == 0) hs *= 2;
    for (; hs >= 1; hs /= 2) {
        const long long per_block = (long long)hs * bs * D * 4;
        if (per_block > kStageCap || hs * bs > 256) continue;
        int nbs = (int)(kStageCap / per_block);
        while (nbs >= 1 && (nbs * bs) % kTile != 0) --nbs;
        if (nbs < 1) continue;
        p->blk_hs = hs;
        p->blk_nbs = nbs;
        p->blk_ok = true;
        break;
    }
    if (!p->blk_ok) return PK_OK;  // the other decode kernel serves this geometry
    int rc;
    switch (D) {
        case 64: rc = blocks_prepare<64>(p); break;
        case 128: rc = blocks_prepare<128>(p); break;
        default: rc = blocks_prepare<256>(p); break;
    }
    if (rc != PK_OK) return rc;
    rc = encode_pool_map3(&p->tmap_kb, p->k_base, p, p->blk_hs * bs);
    if (rc == PK_OK) rc = encode_pool_map3(&p->tmap_vb, p->v_base, p, p->blk_hs * bs);
    return rc;
}

int decode_blocks_chunks_per_cta() { return 2; }  // split partitions a chunk can hold

bool decode_blocks_applies(const pk_pool *p, const AttnArgs &a) {
    return p->blk_ok && a.n_q_heads / p->n_kv_heads <= 8;
}

int launch_decode_blocks(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, bool skip_chunks,
                         bool behind_chunk, cudaStream_t st) {
    switch (p->head_dim) {
        case 64: return blocks_launch<64>(p, a, w, skip_chunks, behind_chunk, st);
        case 128: return blocks_launch<128>(p, a, w, skip_chunks, behind_chunk, st);
        case 256: return blocks_launch<256>(p, a, w, skip_chunks, behind_chunk, st);
        default: return fail(PK_ERR_UNSUPPORTED, "decode path: head_dim %d", p->head_dim);
    }
}

}  // namespace pk
