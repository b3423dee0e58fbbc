// Paged attention on the tensor cores for bf16 pools (head_dim 64/128/256,
// block_size a multiple of 8): decode rows and causal chunked-prefill rows in
// one persistent, warp-specialised kernel per call (per window of at most
// kMaxSeqsPerLaunch sequences).
//
// What is computed ["PagedAttention & Continuous Batching" (study notes),
// "Block tables": the attention kernel gathers through the block table;
// "Batching and PagedAttention", "PagedAttention" item 4 and "Continuous
// batching": one step mixes decodes and prefill chunks]: for query token i of
// sequence b (position p = c_b - q_b + i) and q head h, softmax attention over
// keys 0..p of kv head h / g (g = Hq / Hkv), key j read from physical block
// table_b[j / bs] at slot j % bs.
//
// Decomposition.
//   * Rows.  For one (sequence, kv head) the query rows are the q_b * g pairs
//     (query token, head of the group), numbered token-major; a "row tile" is
//     16 consecutive rows, the M dimension of one m16n8k16 MMA.  A decode
//     with g = 4 fills 4 of the 16 rows; a 512-token chunk fills 128 tiles.
//   * KV tiles.  16 consecutive tokens of the sequence: the N dimension of
//     S = Q K^T (two n8 halves) and the K dimension of O += P V.  Each tile is
//     fetched by TMA from its physical block(s) into a 128-byte-swizzled
//     shared-memory stage, so every ldmatrix below is bank-conflict free.
//   * Work items.  "split" items (sequences with q_b * g <= 16: decodes): one
//     row tile against one partition of the context, processed by ONE
//     consumer warp; partitions are sized so that the batch yields about
//     kItemsPerCta items per resident CTA (flash-decoding-style split-K).
//     The warp that finishes the last partition of a (sequence, kv head)
//     merges all partitions' (O, log-sum-exp) into the output, found by an
//     arrival counter.  "rows" items (chunks): four row tiles, one per
//     consumer warp, against every visible KV tile; each warp masks causally
//     by its own rows.
//   * Planning.  Every CTA derives the same work list from the batch
//     description in shared memory (prefix sums over the window's sequences),
//     so no separate planning kernel runs; items are claimed from a global
//     counter (dynamic scheduling) that the last CTA to finish resets.
//   * Pipeline.  One producer warp claims items two ahead, prefetches each
//     item's block-table entries 32 at a time with one coalesced warp load,
//     stages each consumer warp's Q rows by bulk copy, and streams KV tiles
//     through an NSTAGE-deep ring (full / empty mbarriers per stage); stage
//     metadata names the consumer (one warp, or all four) and marks an
//     item's first and last tile.  Split items of the four warps are
//     interleaved tile by tile.  Consumers run S = Q K^T and O += P V on
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate) with an online softmax in
//     fp32 registers (exp2 with log2(e) folded into the scale, quad shuffles
//     for the row max); they issue no global loads of their own.
//
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel records
// PK_ERR_TIMEOUT in the pool's error word, waits (bounded) for its own TMA
// copies and returns.  Block ids are range-checked before use.
#include "pk_internal.h"

#include <cuda_bf16.h>

#include <algorithm>

namespace pk {
namespace {

constexpr int kMaxSeqsPerLaunch = 512;
constexpr int kPartitionMinTiles = 4;   // smallest split-K partition (64 tokens)
constexpr int kItemsPerCta = 12;         // split-K target: items per resident CTA
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded wait: 2 s
constexpr int kTagAll = 15;             // stage consumed by every consumer warp
constexpr int kTagEnd = -1;              // no more stages
constexpr int kFirst = 1, kLast = 2;     // stage flags

// Workspace header (must start zeroed; every call leaves it zeroed).
struct WsHeader {
    int next_item;  // dynamic scheduler: next item to claim
    int done;       // CTAs finished (the last one resets both fields)
    int pad[62];
};

// One consumer warp's item, written by the producer next to the warp's Q rows.
struct ItemDesc {
    int seq, kvh, tile, kv_begin, kv_end, nparts, part_base, part, pstride, c, qn, qs0, rows;
};

template <int D>
struct TcConfig;
// kConsumers consumer warps + 1 producer warp per CTA.  With 4 warps, two
// CTAs per SM still get 255 registers per thread (a 5-warp CTA is allocated
// as 6 warps, which caps two CTAs at 168 registers and spills the d = 128
// accumulators).
template <>
struct TcConfig<64> {
    static constexpr int kStages = 16, kMinBlocks = 2, kConsumers = 3;
    static constexpr bool kQReg = true;
};
template <>
struct TcConfig<128> {
    static constexpr int kStages = 11, kMinBlocks = 2, kConsumers = 3;
    static constexpr bool kQReg = true;
};
template <>
struct TcConfig<256> {
    static constexpr int kStages = 8, kMinBlocks = 1, kConsumers = 4;
    static constexpr bool kQReg = false;
};
template <int D>
constexpr int threads_of() { return (TcConfig<D>::kConsumers + 1) * 32; }

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

template <int D>
struct Smem {
    static constexpr int kStages = TcConfig<D>::kStages;
    static constexpr int kConsumers = TcConfig<D>::kConsumers;
    static constexpr int kStageBytes = 64 * D;  // K then V: 16 rows x D x 2 bytes each
    static constexpr size_t kRing = 0;
    static constexpr size_t kQStage = kRing + (size_t)kStages * kStageBytes;  // row-major Q rows
    static constexpr size_t kQPriv = kQStage + (size_t)kConsumers * 32 * D;  // swizzled Q (d 256)
    static constexpr size_t kPlan = kQPriv + (TcConfig<D>::kQReg ? 0 : (size_t)kConsumers * 32 * D);
    static constexpr int kPlanLen = kMaxSeqsPerLaunch + 1;
    // plan arrays: split prefix, rows prefix, partial-row prefix, query start
    // lens, context lens
    static constexpr size_t kDesc = kPlan + align_up(5 * (size_t)kPlanLen * 4, 16);
    static constexpr size_t kBars = kDesc + align_up(kConsumers * sizeof(ItemDesc), 16);
    static constexpr size_t kMeta = kBars + (size_t)(2 * kStages + 2 * kConsumers) * 8;
    static constexpr size_t kFlag = kMeta + (size_t)kStages * 16;
    static constexpr size_t kEnd = kFlag + 16;
    static constexpr size_t kBytes = kEnd + 1024;  // + alignment slack
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, int count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits until the phase with the given parity has completed; false after kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Contiguous global -> shared copy (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"((uint64_t)src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Byte offset of the 16-byte chunk holding columns [col, col+8) of row `row`
// in a 16-row tile stored as 64-column panels of 128-byte rows with the
// 128-byte TMA swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t swz(int row, int col) {
    return (uint32_t)((col >> 6) * 2048 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------- parameters
struct TcParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables;
    const int32_t *ctx, *qsl;
    int seq0, nseq;  // this launch's window of sequences
    int max_blocks, n_q_heads, n_kv_heads, group, block_size, box_rows, num_blocks, num_tokens;
    int ncta, cap_rows;  // partial rows the workspace holds
    float scale_log2;
    WsHeader *hdr;
    int *counters;  // per (sequence in the window, kv head): partitions finished
    float *partial_o, *partial_lse;  // [row][D], [row]
    int *err;
};

// An item as the producer sees it (uniform across the producer warp).
struct Item {
    int valid;  // 0: none (queue exhausted)
    int rows;   // 1: rows item (all consumer warps), 0: split item (one warp)
    int b;      // sequence index within the window
    int kvh, group_or_part, nparts, kv_begin, kv_end, part_base, pstride;
};

// Smallest i in [0, n) with pre[i + 1] > idx (pre is an inclusive-scan array
// with pre[0] = 0).
__device__ __forceinline__ int find_seq(const int *pre, int n, int idx) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid + 1] > idx) hi = mid; else lo = mid + 1;
    }
    return lo;
}

template <int D>
__global__ void __launch_bounds__(threads_of<D>(), TcConfig<D>::kMinBlocks)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const TcParams prm) {
    using L = Smem<D>;
    constexpr int S = L::kStages;
    constexpr int kConsumers = TcConfig<D>::kConsumers;
    constexpr int KS = D / 16;  // k-steps of Q K^T and 16-column pairs of P V
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = (uint64_t *)(sm + L::kBars);
    uint64_t *empty = full + S;
    uint64_t *qfull = empty + S;        // [kConsumers] Q rows + descriptor staged
    uint64_t *qempty = qfull + kConsumers;  // [kConsumers] staging area read
    int4 *meta = (int4 *)(sm + L::kMeta);
    volatile int *abort_flag = (volatile int *)(sm + L::kFlag);
    int *split_pre = (int *)(sm + L::kPlan);
    int *rows_pre = split_pre + L::kPlanLen;
    int *prow_pre = rows_pre + L::kPlanLen;
    int *s_qsl = prow_pre + L::kPlanLen;
    int *s_ctx = s_qsl + L::kPlanLen;
    ItemDesc *descs = (ItemDesc *)(sm + L::kDesc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hkv = prm.n_kv_heads, g = prm.group;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        for (int w = 0; w < kConsumers; ++w) {
            mbar_init(&qfull[w], 1);
            mbar_init(&qempty[w], 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kConsumers) {
        // ================================================================ producer warp
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        const int nseq = prm.nseq;
        // ---- plan: the same work list in every CTA
        unsigned long long tiles = 0;
        for (int i = lane; i < nseq; i += 32) {
            const int b = prm.seq0 + i;
            const int s0 = __ldg(prm.qsl + b), s1 = __ldg(prm.qsl + b + 1), c = __ldg(prm.ctx + b);
            const int qn = s1 - s0;
            s_qsl[i] = s0;
            s_ctx[i] = c;
            if (i == nseq - 1) s_qsl[nseq] = s1;
            const bool ok = s0 >= 0 && s1 <= prm.num_tokens && qn >= 1 && c >= qn &&
                            (long long)(c + prm.block_size - 1) / prm.block_size <= prm.max_blocks;
            if (ok && qn * g <= kTile) tiles += (c + kTile - 1) / kTile;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
        __syncwarp();  // s_qsl / s_ctx written by other lanes are read below
        const unsigned long long want = (unsigned long long)prm.ncta * kItemsPerCta;
        unsigned long long P = (tiles * Hkv + want - 1) / want;
        if (P < kPartitionMinTiles) P = kPartitionMinTiles;
        int n_split = 0, n_rows = 0, n_prow = 0;
        for (int attempt = 0; attempt < 8; ++attempt) {
            int run_s = 0, run_r = 0, run_p = 0;
            for (int base = 0; base < nseq; base += 32) {
                const int i = base + lane;
                int ns = 0, nr = 0, np = 0;
                if (i < nseq) {
                    const int c = s_ctx[i], qn = s_qsl[i + 1] - s_qsl[i];
                    const bool ok = s_qsl[i] >= 0 && s_qsl[i + 1] <= prm.num_tokens && qn >= 1 &&
                                    c >= qn &&
                                    (long long)(c + prm.block_size - 1) / prm.block_size <= prm.max_blocks;
                    if (!ok) {
                        if (attempt == 0) record_error(prm.err, PK_ERR_BAD_INDEX);
                    } else if (qn * g <= kTile) {
                        const int kt = (c + kTile - 1) / kTile;
                        const int nparts = (int)(((unsigned long long)kt + P - 1) / P);
                        ns = nparts * Hkv;
                        np = nparts > 1 ? nparts * Hkv * qn * g : 0;
                    } else {
                        const int rtiles = (qn * g + kTile - 1) / kTile;
                        nr = (rtiles + kConsumers - 1) / kConsumers * Hkv;
                    }
                }
                int is = ns, ir = nr, ip = np;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int ys = __shfl_up_sync(0xffffffffu, is, o);
                    const int yr = __shfl_up_sync(0xffffffffu, ir, o);
                    const int yp = __shfl_up_sync(0xffffffffu, ip, o);
                    if (lane >= o) {
                        is += ys;
                        ir += yr;
                        ip += yp;
                    }
                }
                if (i < nseq) {
                    split_pre[i + 1] = run_s + is;
                    rows_pre[i + 1] = run_r + ir;
                    prow_pre[i + 1] = run_p + ip;
                }
                run_s += __shfl_sync(0xffffffffu, is, 31);
                run_r += __shfl_sync(0xffffffffu, ir, 31);
                run_p += __shfl_sync(0xffffffffu, ip, 31);
            }
            n_split = run_s;
            n_rows = run_r;
            n_prow = run_p;
            if (n_prow <= prm.cap_rows) break;
            // more split-K partial rows than the workspace holds (chunks of a few
            // tokens): coarser partitions, finally one partition per sequence
            P = attempt < 6 ? 2 * P : (1ull << 40);
        }
        if (lane == 0) {
            split_pre[0] = 0;
            rows_pre[0] = 0;
            prow_pre[0] = 0;
        }
        __syncwarp();
        const int n_items = n_rows + n_split;

        // ---- item queue: claims are issued two items ahead; the next item's
        // table chunk is loaded when it becomes next, so both latencies hide
        // behind the current item's tiles
        auto claim = [&]() -> int {
            int v = 0;
            if (lane == 0) v = atomicAdd(&prm.hdr->next_item, 1);
            return v;  // valid in lane 0 only; broadcast when used
        };
        auto decode = [&](int idx) -> Item {
            Item it;
            it.valid = idx < n_items;
            it.rows = idx < n_rows;
            it.b = 0;
            it.kvh = it.group_or_part = it.kv_begin = it.kv_end = it.part_base = it.pstride = 0;
            it.nparts = 1;
            if (!it.valid) return it;
            if (it.rows) {
                const int b = find_seq(rows_pre, nseq, idx);
                const int local = idx - rows_pre[b];
                it.b = b;
                it.kvh = local % Hkv;
                it.group_or_part = local / Hkv;
                const int c = s_ctx[b], qn = s_qsl[b + 1] - s_qsl[b];
                const int last_row = min((it.group_or_part + 1) * kConsumers * kTile, qn * g) - 1;
                it.kv_begin = 0;
                it.kv_end = (c - qn + last_row / g) / kTile + 1;
            } else {
                const int j = idx - n_rows;
                const int b = find_seq(split_pre, nseq, j);
                const int local = j - split_pre[b];
                it.b = b;
                it.kvh = local % Hkv;
                it.group_or_part = local / Hkv;
                it.nparts = (split_pre[b + 1] - split_pre[b]) / Hkv;
                const int kt = (s_ctx[b] + kTile - 1) / kTile;
                it.kv_begin = (int)((long long)it.group_or_part * kt / it.nparts);
                it.kv_end = (int)((long long)(it.group_or_part + 1) * kt / it.nparts);
                // partial rows of partition p: part_base + p * pstride .. + rows - 1
                const int rows_b = (s_qsl[b + 1] - s_qsl[b]) * g;
                it.pstride = Hkv * rows_b;
                it.part_base = prow_pre[b] + it.kvh * rows_b;
            }
            return it;
        };
        const int bs = prm.block_size, box = prm.box_rows;
        // this lane's entry of the 32-entry table chunk holding the item's first block
        auto first_chunk = [&](const Item &it) -> int {
            if (!it.valid) return 0;
            const int nblk = (s_ctx[it.b] + bs - 1) / bs;
            const int e = ((it.kv_begin * kTile / bs) & ~31) + lane;
            return e < nblk ? __ldg(prm.tables + (long long)(prm.seq0 + it.b) * prm.max_blocks + e) : 0;
        };
        int ready_idx = __shfl_sync(0xffffffffu, claim(), 0);
        int ready_tab = first_chunk(decode(ready_idx));
        int pending = claim();
        auto pop = [&](int &tab) -> Item {
            const Item it = decode(ready_idx);
            tab = ready_tab;
            ready_idx = __shfl_sync(0xffffffffu, pending, 0);
            ready_tab = first_chunk(decode(ready_idx));
            pending = claim();
            return it;
        };

        // ---- block-table cursor: 32 entries per coalesced warp load, next chunk prefetched
        struct Cursor {
            int base, cur, nxt;
        };
        auto table_of = [&](int seq_abs) { return prm.tables + (long long)seq_abs * prm.max_blocks; };
        auto cursor_start = [&](Cursor &cs, const Item &it, int tab) {
            const int nblk = (s_ctx[it.b] + bs - 1) / bs;
            cs.base = (it.kv_begin * kTile / bs) & ~31;
            cs.cur = tab;
            const int i1 = cs.base + 32 + lane;
            cs.nxt = i1 < nblk ? __ldg(table_of(prm.seq0 + it.b) + i1) : 0;
        };
        auto cursor_get = [&](Cursor &cs, int seq_abs, int nblk, int blk) -> int {
            while (blk >= cs.base + 32) {  // move to the prefetched chunk, prefetch the next
                cs.base += 32;
                cs.cur = cs.nxt;
                const int i1 = cs.base + 32 + lane;
                cs.nxt = i1 < nblk ? __ldg(table_of(seq_abs) + i1) : 0;
            }
            int phys = __shfl_sync(0xffffffffu, cs.cur, blk - cs.base);
            if (phys < 0 || phys >= prm.num_blocks) {
                if (lane == 0) record_error(prm.err, PK_ERR_BAD_INDEX);
                phys = 0;
            }
            return phys;
        };

        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_parity = 0;  // per stage: ever armed, parity of last phase
        uint32_t qphase = 0;                   // per consumer warp: parity bit of qempty waits
        bool ok = true;

        // one KV tile into the next stage, for consumer `tag`; the item is the
        // one described in descs[w] (w = the tag, or 0 for all-warp items)
        auto issue_tile = [&](Cursor &cs, int w, int kt, int tag) {
            if (!ok) return;
            const ItemDesc &d = descs[w];
            const int c = d.c, kvh = d.kvh, seq_abs = d.seq;
            const int flags = (kt == d.kv_begin ? kFirst : 0) | (kt == d.kv_end - 1 ? kLast : 0);
            if (!mbar_wait(&empty[stage], phase ^ 1)) {
                ok = false;
                return;
            }
            const int nblk = (c + bs - 1) / bs;
            int y0 = 0, y1 = 0, nsub = 0;
            for (int t0 = kt * kTile; t0 < kt * kTile + kTile && t0 < c; t0 += box) {
                const int y = (cursor_get(cs, seq_abs, nblk, t0 / bs) * Hkv + kvh) * bs + t0 % bs;
                if (nsub == 0) y0 = y; else y1 = y;
                ++nsub;
            }
            if (lane == 0) {
                meta[stage] = make_int4(tag, kt, flags, 0);
                mbar_arrive_expect_tx(&full[stage], (uint32_t)nsub * 2 * (D / 64) * box * 128);
                uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
                uint8_t *vs = ks + 32 * D;
                for (int sb = 0; sb < nsub; ++sb) {
                    const int y = sb == 0 ? y0 : y1;
#pragma unroll
                    for (int pn = 0; pn < D / 64; ++pn) {
                        tma_load_2d(ks + pn * 2048 + sb * box * 128, &tmk, pn * 64, y, &full[stage]);
                        tma_load_2d(vs + pn * 2048 + sb * box * 128, &tmv, pn * 64, y, &full[stage]);
                    }
                }
            }
            __syncwarp();
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
                stage = 0;
                phase ^= 1;
            }
        };
        // Q rows of row tile `tile` of (b, kvh) and the item descriptor, for warp w
        auto stage_q = [&](int w, const Item &it, int tile) {
            if (!ok) return;
            if (!mbar_wait(&qempty[w], ((qphase >> w) & 1) ^ 1)) {
                ok = false;
                return;
            }
            qphase ^= 1u << w;
            const int b = it.b, c = s_ctx[b], qs0 = s_qsl[b], qn = s_qsl[b + 1] - qs0;
            const int rows_total = qn * g;
            const int r0 = tile * kTile;
            const int nrows = max(0, min(kTile, rows_total - r0));
            if (lane == 0) {
                ItemDesc &d = descs[w];
                d.seq = prm.seq0 + b;
                d.kvh = it.kvh;
                d.tile = nrows > 0 ? tile : -1;
                d.kv_begin = it.kv_begin;
                d.kv_end = it.kv_end;
                d.nparts = it.nparts;
                d.part_base = it.part_base;
                d.part = it.rows ? 0 : it.group_or_part;
                d.pstride = it.pstride;
                d.c = c;
                d.qn = qn;
                d.qs0 = qs0;
                d.rows = rows_total;
                mbar_arrive_expect_tx(&qfull[w], (uint32_t)nrows * D * 2);
            }
            __syncwarp();
            if (nrows > 0) {
                // one contiguous run of heads per query token: lane i copies token t_first + i
                const int t_first = r0 / g, t_last = (r0 + nrows - 1) / g;
                for (int t = t_first + lane; t <= t_last; t += 32) {
                    const int ra = max(r0, t * g), rb = min(r0 + nrows, (t + 1) * g);
                    const __nv_bfloat16 *src =
                        prm.q + ((long long)(qs0 + t) * prm.n_q_heads + it.kvh * g + (ra - t * g)) * D;
                    bulk_load(sm + L::kQStage + (size_t)w * 32 * D + (size_t)(ra - r0) * D * 2, src,
                              (uint32_t)(rb - ra) * D * 2, &qfull[w]);
                }
            }
            __syncwarp();
        };

        // ---- rows items: all four consumer warps on every tile
        while (ok && ready_idx < n_rows) {
            int tab;
            const Item it = pop(tab);
            for (int w = 0; w < kConsumers; ++w) stage_q(w, it, it.group_or_part * kConsumers + w);
            Cursor cs;
            cursor_start(cs, it, tab);
            for (int kt = it.kv_begin; kt < it.kv_end && ok; ++kt) issue_tile(cs, 0, kt, kTagAll);
        }
        // ---- split items: one per consumer warp, tiles interleaved round-robin
        Cursor cur_w[kConsumers];
        int kt_w[kConsumers], ke_w[kConsumers];
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) kt_w[w] = ke_w[w] = 0;
        bool exhausted = ready_idx >= n_items;
        while (ok) {
            bool any = false;
#pragma unroll
            for (int w = 0; w < kConsumers; ++w) {
                if (kt_w[w] >= ke_w[w] && !exhausted) {
                    int tab;
                    const Item it = pop(tab);
                    stage_q(w, it, 0);
                    cursor_start(cur_w[w], it, tab);
                    kt_w[w] = it.kv_begin;
                    ke_w[w] = it.kv_end;
                    exhausted = ready_idx >= n_items;
                }
                if (kt_w[w] < ke_w[w]) {
                    issue_tile(cur_w[w], w, kt_w[w], w);
                    ++kt_w[w];
                    any = true;
                }
            }
            if (!any && exhausted) break;
        }
        // ---- end marker
        if (ok && mbar_wait(&empty[stage], phase ^ 1)) {
            if (lane == 0) {
                meta[stage] = make_int4(kTagEnd, 0, 0, 0);
                mbar_arrive(&full[stage]);
            }
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        } else {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        // never leave with a copy still writing into this CTA's shared memory
        if (lane == 0)
            for (int s = 0; s < S; ++s)
                if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1);
        __syncwarp();
    } else {
        // ================================================================ consumer warps
        const int w = warp;
        const int qr = lane >> 2;       // fragment row (and row + 8)
        const int qc = (lane & 3) * 2;  // fragment column pair
        const int mi = lane >> 3, rr = lane & 7;
        const int k_row = (mi >> 1) * 8 + rr, k_col = (mi & 1) * 8;  // K (B of Q K^T)
        const int v_row = (mi & 1) * 8 + rr, v_col = (mi >> 1) * 8;  // V (B of P V, transposed)
        const int q_row = (mi & 1) * 8 + rr, q_col = (mi >> 1) * 8;  // Q (A of Q K^T)
        const int Hq = prm.n_q_heads;
        const uint8_t *qstage = sm + L::kQStage + (size_t)w * 32 * D;
        uint8_t *qpriv = sm + L::kQPriv + (size_t)w * 32 * D;

        int stage = 0;
        uint32_t phase = 0, qph = 0;
        int d_seq = 0, d_kvh = 0, d_nparts = 1, d_row = 0, d_qs0 = 0, d_rows = 0, d_base = 0,
            d_pstride = 0;
        bool active = false;
        int c = 0, max_lim = 0, lim0 = 0, lim1 = 0;
        long long orow0 = -1, orow1 = -1;  // output rows, -1 = not a query row
        uint32_t qf[TcConfig<D>::kQReg ? KS : 1][4];
        float o[D / 8][4];
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        bool ok = true;

        auto begin_item = [&]() {
            if (!mbar_wait(&qfull[w], qph)) {
                ok = false;
                return;
            }
            qph ^= 1;
            const ItemDesc &dsc = descs[w];
            active = dsc.tile >= 0;
            c = dsc.c;
            const int rows = dsc.rows, qn = dsc.qn;
            d_seq = dsc.seq;
            d_kvh = dsc.kvh;
            d_nparts = dsc.nparts;
            d_base = dsc.part_base;
            d_pstride = dsc.pstride;
            d_row = dsc.part_base + dsc.part * dsc.pstride;
            d_qs0 = dsc.qs0;
            d_rows = rows;
            const int tile = max(dsc.tile, 0);
            const int r0 = tile * kTile + qr, r1 = r0 + 8;
            // rows past the last query row compute garbage that is never written
            lim0 = r0 < rows ? c - qn + r0 / g : c - 1;
            lim1 = r1 < rows ? c - qn + r1 / g : c - 1;
            max_lim = c - qn + (min(tile * kTile + kTile, rows) - 1) / g;
            orow0 = active && r0 < rows ? (long long)(d_qs0 + r0 / g) * Hq + d_kvh * g + r0 % g : -1;
            orow1 = active && r1 < rows ? (long long)(d_qs0 + r1 / g) * Hq + d_kvh * g + r1 % g : -1;
            const int nvalid = active ? min(kTile, rows - tile * kTile) : 0;
            if constexpr (TcConfig<D>::kQReg) {
                const uint8_t *q0 = qstage + qr * D * 2, *q1 = qstage + (qr + 8) * D * 2;
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    const int col = (ks * 16 + qc) * 2;
                    qf[ks][0] = qr < nvalid ? *(const uint32_t *)(q0 + col) : 0u;
                    qf[ks][1] = qr + 8 < nvalid ? *(const uint32_t *)(q1 + col) : 0u;
                    qf[ks][2] = qr < nvalid ? *(const uint32_t *)(q0 + col + 16) : 0u;
                    qf[ks][3] = qr + 8 < nvalid ? *(const uint32_t *)(q1 + col + 16) : 0u;
                }
            } else {
                for (int ch = lane; ch < 16 * (D / 8); ch += 32) {
                    const int row = ch / (D / 8), col = (ch % (D / 8)) * 8;
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (row < nvalid) v = *(const uint4 *)(qstage + (row * D + col) * 2);
                    *(uint4 *)(qpriv + swz(row, col)) = v;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[w]);
#pragma unroll
            for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
        };

        auto finish_item = [&]() {
            if (!active) return;
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
            if (d_nparts <= 1) {
                if (orow0 >= 0) {
                    __nv_bfloat16 *dst = prm.out + orow0 * D;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n)
                        *(uint32_t *)(dst + n * 8 + qc) = pack_bf16(o[n][0] * inv0, o[n][1] * inv0);
                }
                if (orow1 >= 0) {
                    __nv_bfloat16 *dst = prm.out + orow1 * D;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n)
                        *(uint32_t *)(dst + n * 8 + qc) = pack_bf16(o[n][2] * inv1, o[n][3] * inv1);
                }
                return;
            }
            // split-K partition: normalised O and log2-sum-exp of the valid rows
            float *po = prm.partial_o + (size_t)d_row * D;
            if (orow0 >= 0)
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *(float2 *)(po + qr * D + n * 8 + qc) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
            if (orow1 >= 0)
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *(float2 *)(po + (qr + 8) * D + n * 8 + qc) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
            if ((lane & 3) == 0) {
                float *pl = prm.partial_lse + (size_t)d_row;
                if (orow0 >= 0) pl[qr] = l0 > 0.f ? m0 + __log2f(l0) : -INFINITY;
                if (orow1 >= 0) pl[qr + 8] = l1 > 0.f ? m1 + __log2f(l1) : -INFINITY;
            }
            __threadfence();
            __syncwarp();
            int prev = 0;
            int *cnt = prm.counters + (size_t)(d_seq - prm.seq0) * Hkv + d_kvh;
            if (lane == 0) prev = atomicAdd(cnt, 1);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev != d_nparts - 1) return;
            // last partition of (sequence, kv head): merge all partitions into the output
            __threadfence();
            const int nrows = min(kTile, d_rows);
            for (int idx = lane; idx < nrows * (D / 4); idx += 32) {
                const int row = idx / (D / 4), c4 = idx % (D / 4);
                float M = -INFINITY;
                for (int p = 0; p < d_nparts; ++p)
                    M = fmaxf(M, __ldcg(prm.partial_lse + (size_t)(d_base + p * d_pstride) + row));
                float den = 0.f;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int p = 0; p < d_nparts; ++p) {
                    const size_t pr = (size_t)(d_base + p * d_pstride) + row;
                    const float lse = __ldcg(prm.partial_lse + pr);
                    const float wgt = lse == -INFINITY ? 0.f : fast_exp2(lse - M);
                    const float4 x = __ldcg((const float4 *)(prm.partial_o + pr * D) + c4);
                    den += wgt;
                    acc.x += wgt * x.x;
                    acc.y += wgt * x.y;
                    acc.z += wgt * x.z;
                    acc.w += wgt * x.w;
                }
                const float inv = den > 0.f ? 1.f / den : 0.f;
                const long long orow = (long long)(d_qs0 + row / g) * Hq + d_kvh * g + row % g;
                uint2 pk;
                pk.x = pack_bf16(acc.x * inv, acc.y * inv);
                pk.y = pack_bf16(acc.z * inv, acc.w * inv);
                *(uint2 *)(prm.out + orow * D + c4 * 4) = pk;
            }
            if (lane == 0) *cnt = 0;  // leave the counter zeroed for the next call
        };

        auto compute_tile = [&](int kt, uint8_t *ks, uint8_t *vs, bool zero_tail) {
            const int valid = c - kt * kTile;  // tokens of this tile inside the context
            if (valid < kTile && zero_tail) {
                // tail tile: clear V rows past the context (stale or never-written slots)
                for (int ch = lane; ch < (kTile - valid) * (D / 8); ch += 32) {
                    const int row = valid + ch / (D / 8), col = (ch % (D / 8)) * 8;
                    *(uint4 *)(vs + swz(row, col)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
                __syncwarp();
            }
            const uint32_t ka = smem_u32(ks), va = smem_u32(vs), qa = smem_u32(qpriv);
            float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a0, a1, a2, a3;
                if constexpr (TcConfig<D>::kQReg) {
                    a0 = qf[kk][0];
                    a1 = qf[kk][1];
                    a2 = qf[kk][2];
                    a3 = qf[kk][3];
                } else {
                    ldsm_x4(qa + swz(q_row, kk * 16 + q_col), a0, a1, a2, a3);
                }
                uint32_t b0, b1, b2, b3;
                ldsm_x4(ka + swz(k_row, kk * 16 + k_col), b0, b1, b2, b3);
                mma_bf16(sc[0], a0, a1, a2, a3, b0, b1);
                mma_bf16(sc[1], a0, a1, a2, a3, b2, b3);
            }
            // scores in the log2 domain, causal / context mask by key position
            const int key0 = kt * kTile + qc;
            const bool full_tile = kt * kTile + kTile - 1 <= min(lim0, lim1);
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float s = sc[nt][i] * prm.scale_log2;
                    if (!full_tile) {
                        const int key = key0 + nt * 8 + (i & 1);
                        if (key > (i < 2 ? lim0 : lim1)) s = -INFINITY;
                    }
                    sc[nt][i] = s;
                    if (i < 2) mx0 = fmaxf(mx0, s); else mx1 = fmaxf(mx1, s);
                }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
            const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
            const float b0 = mn0 == -INFINITY ? 0.f : mn0, b1 = mn1 == -INFINITY ? 0.f : mn1;
            const float al0 = fast_exp2(m0 - b0), al1 = fast_exp2(m1 - b1);
            m0 = mn0;
            m1 = mn1;
            float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                sc[nt][0] = fast_exp2(sc[nt][0] - b0);
                sc[nt][1] = fast_exp2(sc[nt][1] - b0);
                sc[nt][2] = fast_exp2(sc[nt][2] - b1);
                sc[nt][3] = fast_exp2(sc[nt][3] - b1);
                ps0 += sc[nt][0] + sc[nt][1];
                ps1 += sc[nt][2] + sc[nt][3];
            }
            l0 = l0 * al0 + ps0;
            l1 = l1 * al1 + ps1;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= al0;
                o[n][1] *= al0;
                o[n][2] *= al1;
                o[n][3] *= al1;
            }
            const uint32_t p0 = pack_bf16(sc[0][0], sc[0][1]), p1 = pack_bf16(sc[0][2], sc[0][3]);
            const uint32_t p2 = pack_bf16(sc[1][0], sc[1][1]), p3 = pack_bf16(sc[1][2], sc[1][3]);
#pragma unroll
            for (int np = 0; np < KS; ++np) {
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(va + swz(v_row, np * 16 + v_col), v0, v1, v2, v3);
                mma_bf16(o[2 * np], p0, p1, p2, p3, v0, v1);
                mma_bf16(o[2 * np + 1], p0, p1, p2, p3, v2, v3);
            }
        };

        for (;;) {
            if (!mbar_wait(&full[stage], phase)) {
                ok = false;
                break;
            }
            const int4 mt = meta[stage];
            if (mt.x == kTagEnd) break;
            if (mt.x == w || mt.x == kTagAll) {
                if (mt.z & kFirst) begin_item();
                if (!ok) break;
                if (active && mt.y * kTile <= max_lim) {
                    uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
                    compute_tile(mt.y, ks, ks + 32 * D, true);
                }
                if (mt.z & kLast) finish_item();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == S) {
                stage = 0;
                phase ^= 1;
            }
            if (*abort_flag) break;
        }
        if (!ok) {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    }

    // the last CTA to finish resets the work counter for the next call
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int d = atomicAdd(&prm.hdr->done, 1);
        if (d == (int)gridDim.x - 1) {
            prm.hdr->next_item = 0;
            prm.hdr->done = 0;
            __threadfence();
        }
    }
}

}  // namespace
}  // namespace pk

namespace pk {
namespace {

// Workspace: header | counters (fixed size) | partial lse | partial O.  The
// header and counters sit at offsets that do not depend on the batch, so the
// zeros every call leaves there stay valid when the next call's batch differs.
struct WsLayout {
    size_t counters, partial_lse, partial_o, total;
    int cap_rows;
};

WsLayout ws_layout(const pk_pool *p, int num_seqs, int n_q_heads) {
    WsLayout L{};
    const int Hkv = p->n_kv_heads, D = p->head_dim;
    const int g = std::max(1, n_q_heads / Hkv);
    // split items: at most Hkv per sequence plus the ~kItemsPerCta per CTA that
    // split-K adds; a decode item has g partial rows (the planner coarsens the
    // partitions if a batch needs more)
    const long long items = (long long)Hkv * std::min(num_seqs, kMaxSeqsPerLaunch) +
                            (long long)p->tc_ctas * kItemsPerCta;
    L.cap_rows = (int)std::min<long long>(items * std::min(g, kTile), 1LL << 30);
    size_t off = align_up(sizeof(WsHeader), 256);
    L.counters = off;
    off = align_up(off + (size_t)kMaxSeqsPerLaunch * Hkv * sizeof(int), 256);
    L.partial_lse = off;
    off = align_up(off + (size_t)L.cap_rows * sizeof(float), 256);
    L.partial_o = off;
    off = align_up(off + (size_t)L.cap_rows * D * sizeof(float), 256);
    L.total = off;
    return L;
}

template <int D>
int prepare(pk_pool *p) {
    const int smem = (int)Smem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "set attention smem size");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_tc_kernel<D>, threads_of<D>(), smem);
    if (e != cudaSuccess) return cuda_fail(e, "attention occupancy");
    if (per_sm < 1) return fail(PK_ERR_UNSUPPORTED, "attention kernel does not fit on an SM");
    p->tc_ctas = per_sm * p->sm_count;
    return PK_OK;
}

template <int D>
int launch(const pk_pool *p, const AttnArgs &a, const WsLayout &L, cudaStream_t st) {
    uint8_t *ws = (uint8_t *)a.workspace;
    TcParams tp;
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
    tp.box_rows = p->block_size % kTile == 0 ? kTile : 8;
    tp.num_blocks = p->num_blocks;
    tp.num_tokens = a.num_tokens;
    tp.ncta = p->tc_ctas;
    tp.cap_rows = L.cap_rows;
    tp.scale_log2 = a.scale * 1.4426950408889634f;
    tp.hdr = (WsHeader *)ws;
    tp.counters = (int *)(ws + L.counters);
    tp.partial_o = (float *)(ws + L.partial_o);
    tp.partial_lse = (float *)(ws + L.partial_lse);
    tp.err = p->d_err;
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        tp.seq0 = s0;
        tp.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        attention_tc_kernel<D><<<p->tc_ctas, threads_of<D>(), Smem<D>::kBytes, st>>>(p->tmap_k, p->tmap_v, tp);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "tensor-core attention launch");
}

}  // namespace

size_t tc_workspace_bytes(const pk_pool *p, int num_seqs, int num_tokens, int n_q_heads,
                          int /*max_blocks_per_seq*/) {
    (void)num_tokens;
    return ws_layout(p, num_seqs, n_q_heads).total;
}

int tc_prepare_pool(pk_pool *p) {
    switch (p->head_dim) {
        case 64: return prepare<64>(p);
        case 128: return prepare<128>(p);
        case 256: return prepare<256>(p);
        default: return fail(PK_ERR_UNSUPPORTED, "tensor-core path: head_dim %d", p->head_dim);
    }
}

int launch_attention_tc(const pk_pool *p, const AttnArgs &a, cudaStream_t st) {
    const WsLayout L = ws_layout(p, a.num_seqs, a.n_q_heads);
    if (a.workspace_bytes < L.total || a.workspace == nullptr)
        return fail(PK_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", a.workspace_bytes, L.total);
    if (((uintptr_t)a.workspace & 255) != 0)
        return fail(PK_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    switch (p->head_dim) {
        case 64: return launch<64>(p, a, L, st);
        case 128: return launch<128>(p, a, L, st);
        case 256: return launch<256>(p, a, L, st);
        default: return fail(PK_ERR_UNSUPPORTED, "tensor-core path: head_dim %d", p->head_dim);
    }
}

}  // namespace pk
