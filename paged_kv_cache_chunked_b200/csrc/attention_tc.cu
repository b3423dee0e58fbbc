// Paged attention on the tensor cores for bf16 pools (head_dim 64/128/256,
// block_size a multiple of 8): decode rows and causal chunked-prefill rows in
// one persistent, warp-specialised kernel, plus a device-side work planner
// and a split-K reduce.
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
//   * Rows.  For one (sequence, kv head) the query rows are the q_b * g
//     pairs (query token, head of the group), numbered token-major; a "row
//     tile" is 16 consecutive rows: the M dimension of one m16n8k16 MMA.
//     A decode step with g = 4 fills 4 of the 16 rows; a 512-token chunk
//     fills 128 row tiles.
//   * KV tiles.  16 consecutive tokens of the sequence: the N dimension of
//     S = Q K^T (two n8 halves) and the K dimension of O += P V.  Each tile
//     is fetched by TMA from its physical block(s) into a 128-byte-swizzled
//     shared-memory stage, so every ldmatrix below is bank-conflict free.
//   * Work items.  "split" items: one row tile (sequences with q_b * g <= 16,
//     i.e. decodes) and a range of KV tiles; the four consumer warps take
//     every fourth tile of the range and merge their (max, sum, O) at the
//     end; ranges are partitions of the context sized so that the whole
//     batch yields about eight items per resident CTA (flash-decoding
//     style), and a separate reduce kernel combines the partitions.
//     "rows" items: four row tiles (one per consumer warp) against all
//     visible KV tiles; each warp masks causally by its own rows.
//   * Pipeline.  One producer warp claims items from a global counter and
//     streams their KV tiles through an NSTAGE-deep ring (mbarrier full /
//     empty per stage, stage metadata naming the item and tile).  Consumer
//     warps run S = Q K^T and O += P V on mma.sync m16n8k16 (bf16 in, fp32
//     accumulate) with an online softmax in fp32 registers (exp2 with
//     log2(e) folded into the scale, quad shuffles for the row max).
//
// Every wait is bounded (2 s of %globaltimer); on expiry the kernel records
// PK_ERR_TIMEOUT in the pool's error word, waits (bounded) for its own TMA
// copies and returns.  Block ids are range-checked before use.
#include "pk_internal.h"

#include <cuda_bf16.h>

#include <algorithm>

namespace pk {
namespace {

constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kPartitionMinTiles = 4;   // smallest split-K partition (64 tokens)
constexpr int kItemsPerCta = 8;          // split-K target: items per resident CTA
constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded wait: 2 s

struct WorkItem {
    int seq, kvh, row_tile, kv_begin, kv_end, partial, pad0, pad1;
};
struct ReduceItem {
    int seq, kvh, first_partial, n_parts;
};
struct WsHeader {
    int n_rows_items;
    int n_split_items;
    int n_reduce;
    int next_item;  // dynamic scheduler: next item to claim
    int pad[12];
};

struct WsLayout {
    size_t items_rows, items_split, reduce, partial_o, partial_lse, total;
    int cap_rows, cap_split, cap_reduce;
};

template <int D>
struct TcConfig;
template <>
struct TcConfig<64> {
    static constexpr int kStages = 16, kMinBlocks = 2;
    static constexpr bool kQReg = true;
};
template <>
struct TcConfig<128> {
    static constexpr int kStages = 10, kMinBlocks = 2;
    static constexpr bool kQReg = true;
};
template <>
struct TcConfig<256> {
    static constexpr int kStages = 8, kMinBlocks = 1;
    static constexpr bool kQReg = false;
};

template <int D>
constexpr size_t smem_bytes() {
    return 1024 /* alignment slack */ + (size_t)TcConfig<D>::kStages * 64 * D  // ring
           + (size_t)(kConsumers - 1) * 16 * D * 4                           // merge O
           + (size_t)(kConsumers - 1) * 16 * 2 * 4                           // merge m, l
           + (TcConfig<D>::kQReg ? 0 : (size_t)kConsumers * 32 * D)          // Q tiles
           + (size_t)(2 * TcConfig<D>::kStages + 2) * 8                      // mbarriers
           + (size_t)TcConfig<D>::kStages * 16 + 16;                         // metadata, flag
}

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

// ---------------------------------------------------------------- planner
struct PlanArgs {
    const int32_t *ctx, *qsl;
    int num_seqs, num_tokens, group, n_kv_heads, block_size, max_blocks, ncta;
    int cap_rows, cap_split, cap_reduce;
    WsHeader *hdr;
    WorkItem *items_rows, *items_split;
    ReduceItem *reduce;
    int *err;
};

__device__ bool seq_shape(const PlanArgs &a, int b, int &q, int &c) {
    const int s0 = a.qsl[b], s1 = a.qsl[b + 1];
    q = s1 - s0;
    c = a.ctx[b];
    return s0 >= 0 && s1 <= a.num_tokens && q >= 1 && c >= q &&
           (int64_t)(c + a.block_size - 1) / a.block_size <= a.max_blocks;
}

// Exclusive prefix sum over the 1024 threads of the block; *total = sum.
__device__ int block_scan(int v, int *total, int *sh) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[w] = x;
    __syncthreads();
    if (w == 0) {
        int s = sh[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        sh[lane] = s;
    }
    __syncthreads();
    const int res = (w ? sh[w - 1] : 0) + x - v;
    *total = sh[31];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(1024) plan_kernel(PlanArgs a) {
    __shared__ int sh[32];
    __shared__ unsigned long long s_tiles;
    if (threadIdx.x == 0) s_tiles = 0;
    __syncthreads();
    const int Hkv = a.n_kv_heads, g = a.group;
    // pass 1: KV tiles of all split sequences -> partition size
    unsigned long long tiles = 0;
    for (int b = threadIdx.x; b < a.num_seqs; b += blockDim.x) {
        int q, c;
        if (seq_shape(a, b, q, c) && q * g <= kTile) tiles += (c + kTile - 1) / kTile;
    }
    atomicAdd(&s_tiles, tiles);
    __syncthreads();
    const unsigned long long want = (unsigned long long)a.ncta * kItemsPerCta;
    unsigned long long P = (s_tiles * Hkv + want - 1) / want;
    if (P < kPartitionMinTiles) P = kPartitionMinTiles;

    // pass 2: items
    int base_r = 0, base_s = 0, base_red = 0, base_p = 0;
    for (int start = 0; start < a.num_seqs; start += blockDim.x) {
        const int b = start + threadIdx.x;
        int q = 0, c = 0, nr = 0, ns = 0, nred = 0, npart = 0, nparts = 0, ngroups = 0, kt = 0;
        bool split = false;
        if (b < a.num_seqs) {
            if (seq_shape(a, b, q, c)) {
                kt = (c + kTile - 1) / kTile;
                split = q * g <= kTile;
                if (split) {
                    nparts = (int)(((unsigned long long)kt + P - 1) / P);
                    ns = nparts * Hkv;
                    if (nparts > 1) {
                        npart = nparts * Hkv;
                        nred = Hkv;
                    }
                } else {
                    const int rtiles = (q * g + kTile - 1) / kTile;
                    ngroups = (rtiles + kConsumers - 1) / kConsumers;
                    nr = ngroups * Hkv;
                }
            } else {
                record_error(a.err, PK_ERR_BAD_INDEX);
            }
        }
        int tot_r, tot_s, tot_red, tot_p;
        const int o_r = base_r + block_scan(nr, &tot_r, sh);
        const int o_s = base_s + block_scan(ns, &tot_s, sh);
        const int o_red = base_red + block_scan(nred, &tot_red, sh);
        const int o_p = base_p + block_scan(npart, &tot_p, sh);
        if (o_r + nr > a.cap_rows || o_s + ns > a.cap_split || o_red + nred > a.cap_reduce) {
            record_error(a.err, PK_ERR_BAD_INDEX);  // cannot happen with host-sized caps
        } else if (split) {
            for (int p = 0; p < nparts; ++p) {
                const int kb = (int)((long long)p * kt / nparts);
                const int ke = (int)((long long)(p + 1) * kt / nparts);
                for (int h = 0; h < Hkv; ++h) {
                    WorkItem it;
                    it.seq = b;
                    it.kvh = h;
                    it.row_tile = 0;
                    it.kv_begin = kb;
                    it.kv_end = ke;
                    it.partial = nparts > 1 ? o_p + h * nparts + p : -1;
                    it.pad0 = it.pad1 = 0;
                    a.items_split[o_s + p * Hkv + h] = it;
                }
            }
            if (nparts > 1)
                for (int h = 0; h < Hkv; ++h) {
                    ReduceItem r;
                    r.seq = b;
                    r.kvh = h;
                    r.first_partial = o_p + h * nparts;
                    r.n_parts = nparts;
                    a.reduce[o_red + h] = r;
                }
        } else if (ngroups > 0) {
            const int rows = q * g;
            for (int gi = 0; gi < ngroups; ++gi) {
                const int rt = gi * kConsumers;
                const int last_row = min((rt + kConsumers) * kTile, rows) - 1;
                const int lim = c - q + last_row / g;  // last visible key of the group
                for (int h = 0; h < Hkv; ++h) {
                    WorkItem it;
                    it.seq = b;
                    it.kvh = h;
                    it.row_tile = rt;
                    it.kv_begin = 0;
                    it.kv_end = lim / kTile + 1;
                    it.partial = -1;
                    it.pad0 = it.pad1 = 0;
                    a.items_rows[o_r + gi * Hkv + h] = it;
                }
            }
        }
        base_r += tot_r;
        base_s += tot_s;
        base_red += tot_red;
        base_p += tot_p;
    }
    if (threadIdx.x == 0) {
        a.hdr->n_rows_items = min(base_r, a.cap_rows);
        a.hdr->n_split_items = min(base_s, a.cap_split);
        a.hdr->n_reduce = min(base_red, a.cap_reduce);
        a.hdr->next_item = 0;
    }
}

// ---------------------------------------------------------------- attention
struct TcParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables;
    const int32_t *ctx, *qsl;
    int max_blocks, n_q_heads, n_kv_heads, group, block_size, box_rows, num_blocks;
    float scale_log2;
    WsHeader *hdr;
    const WorkItem *items_rows, *items_split;
    float *partial_o, *partial_lse;
    int *err;
};

template <int D>
struct Smem {
    static constexpr int kStages = TcConfig<D>::kStages;
    static constexpr int kStageBytes = 64 * D;  // K then V, 16 rows x D x 2 bytes each
    static constexpr size_t kRing = 0;
    static constexpr size_t kMergeO = kRing + (size_t)kStages * kStageBytes;
    static constexpr size_t kMergeML = kMergeO + (size_t)(kConsumers - 1) * 16 * D * 4;
    static constexpr size_t kQ = kMergeML + (size_t)(kConsumers - 1) * 16 * 2 * 4;
    static constexpr size_t kBars =
        kQ + (TcConfig<D>::kQReg ? 0 : (size_t)kConsumers * 32 * D);
    static constexpr size_t kMeta = kBars + (size_t)(2 * kStages + 2) * 8;
    static constexpr size_t kFlag = kMeta + (size_t)kStages * 16;
    static constexpr size_t kEnd = kFlag + 16;
};

template <int D>
__global__ void __launch_bounds__(kThreads, TcConfig<D>::kMinBlocks)
attention_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const TcParams prm) {
    using L = Smem<D>;
    constexpr int S = L::kStages;
    constexpr int KS = D / 16;  // k-steps of Q K^T and 16-column pairs of P V
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = (uint64_t *)(sm + L::kBars);
    uint64_t *empty = full + S;
    uint64_t *mfull = empty + S;   // merge buffer written by warps 1..3
    uint64_t *mempty = mfull + 1;  // merge buffer read by warp 0
    int4 *meta = (int4 *)(sm + L::kMeta);
    volatile int *abort_flag = (volatile int *)(sm + L::kFlag);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        mbar_init(mfull, kConsumers - 1);
        mbar_init(mempty, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int n_rows_items = prm.hdr->n_rows_items;
    const int n_items = n_rows_items + prm.hdr->n_split_items;

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        const int bs = prm.block_size, box = prm.box_rows, Hkv = prm.n_kv_heads;
        const uint32_t box_bytes = (uint32_t)box * 128;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_parity = 0;  // per stage: ever armed, parity of last arm
        bool ok = true;
        for (;;) {
            const int idx = atomicAdd(&prm.hdr->next_item, 1);
            if (idx >= n_items) break;
            const WorkItem it = idx < n_rows_items ? prm.items_rows[idx]
                                                   : prm.items_split[idx - n_rows_items];
            const int c = __ldg(prm.ctx + it.seq);
            const int32_t *table = prm.tables + (int64_t)it.seq * prm.max_blocks;
            for (int kt = it.kv_begin; kt < it.kv_end && ok; ++kt) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) {
                    ok = false;
                    break;
                }
                meta[stage] = make_int4(idx, kt, 0, 0);
                int ys[2];
                int nsub = 0;
                for (int t0 = kt * kTile; t0 < kt * kTile + kTile && t0 < c; t0 += box) {
                    int phys = __ldg(table + t0 / bs);
                    if (phys < 0 || phys >= prm.num_blocks) {
                        record_error(prm.err, PK_ERR_BAD_INDEX);
                        phys = 0;
                    }
                    ys[nsub++] = (phys * Hkv + it.kvh) * bs + t0 % bs;
                }
                mbar_arrive_expect_tx(&full[stage], (uint32_t)nsub * 2 * (D / 64) * box_bytes);
                uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
                uint8_t *vs = ks + 32 * D;
                for (int sb = 0; sb < nsub; ++sb)
#pragma unroll
                    for (int pn = 0; pn < D / 64; ++pn) {
                        tma_load_2d(ks + pn * 2048 + sb * box_bytes, &tmk, pn * 64, ys[sb], &full[stage]);
                        tma_load_2d(vs + pn * 2048 + sb * box_bytes, &tmv, pn * 64, ys[sb], &full[stage]);
                    }
                armed |= 1u << stage;
                armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) break;
        }
        if (ok && mbar_wait(&empty[stage], phase ^ 1)) {
            meta[stage] = make_int4(-1, 0, 0, 0);
            mbar_arrive(&full[stage]);
            // the end marker completes a phase of this stage's barrier too
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        } else {
            record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        // never leave with a TMA copy still writing into this CTA's shared memory
        for (int s = 0; s < S; ++s)
            if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1);
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp;
    const int qr = lane >> 2;      // fragment row (and row + 8)
    const int qc = (lane & 3) * 2; // fragment column pair
    const int mi = lane >> 3, rr = lane & 7;
    // per-lane ldmatrix row/column offsets
    const int k_row = (mi >> 1) * 8 + rr, k_col = (mi & 1) * 8;  // K (B of Q K^T)
    const int v_row = (mi & 1) * 8 + rr, v_col = (mi >> 1) * 8;  // V (B of P V, transposed)
    const int q_row = (mi & 1) * 8 + rr, q_col = (mi >> 1) * 8;  // Q (A of Q K^T)

    const int g = prm.group, Hq = prm.n_q_heads;
    float *merge_o = (float *)(sm + L::kMergeO);
    float *merge_ml = (float *)(sm + L::kMergeML);
    uint8_t *qsm = sm + L::kQ + (size_t)w * 32 * D;

    int stage = 0;
    uint32_t phase = 0, mphase = 0;
    int cur = -1;
    bool rows_mode = false, active = false;
    int seq = 0, c = 0, kvb = 0, partial = -1, max_lim = 0, lim0 = 0, lim1 = 0;
    int64_t orow0 = -1, orow1 = -1;  // output rows (element offsets / D), -1 = none
    uint32_t qf[TcConfig<D>::kQReg ? KS : 1][4];
    float o[D / 8][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    bool ok = true;

    auto begin_item = [&](int idx) {
        rows_mode = idx < n_rows_items;
        const WorkItem it = rows_mode ? prm.items_rows[idx] : prm.items_split[idx - n_rows_items];
        seq = it.seq;
        kvb = it.kv_begin;
        partial = it.partial;
        c = __ldg(prm.ctx + seq);
        const int qs0 = __ldg(prm.qsl + seq);
        const int qn = __ldg(prm.qsl + seq + 1) - qs0;
        const int rows = qn * g;
        const int tile = rows_mode ? it.row_tile + w : 0;
        active = tile * kTile < rows;
        const int r0 = tile * kTile + qr, r1 = r0 + 8;
        // rows past the sequence's last query row compute garbage that is never written
        lim0 = r0 < rows ? c - qn + r0 / g : c - 1;
        lim1 = r1 < rows ? c - qn + r1 / g : c - 1;
        max_lim = c - qn + (min(tile * kTile + kTile, rows) - 1) / g;
        orow0 = r0 < rows ? (int64_t)(qs0 + r0 / g) * Hq + it.kvh * g + r0 % g : -1;
        orow1 = r1 < rows ? (int64_t)(qs0 + r1 / g) * Hq + it.kvh * g + r1 % g : -1;
        const __nv_bfloat16 *q0 = orow0 >= 0 ? prm.q + orow0 * D : nullptr;
        const __nv_bfloat16 *q1 = orow1 >= 0 ? prm.q + orow1 * D : nullptr;
        if constexpr (TcConfig<D>::kQReg) {
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int col = ks * 16 + qc;
                qf[ks][0] = q0 ? __ldg((const uint32_t *)(q0 + col)) : 0u;
                qf[ks][1] = q1 ? __ldg((const uint32_t *)(q1 + col)) : 0u;
                qf[ks][2] = q0 ? __ldg((const uint32_t *)(q0 + col + 8)) : 0u;
                qf[ks][3] = q1 ? __ldg((const uint32_t *)(q1 + col + 8)) : 0u;
            }
        } else {
            // 16 rows x D into the swizzled per-warp tile: lane handles 16-byte chunks
            for (int ch = lane; ch < 16 * (D / 8); ch += 32) {
                const int row = ch / (D / 8), col = (ch % (D / 8)) * 8;
                const int rg = tile * kTile + row;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (rg < rows)
                    v = __ldg((const uint4 *)(prm.q +
                                              ((int64_t)(qs0 + rg / g) * Hq + it.kvh * g + rg % g) * D +
                                              col));
                *(uint4 *)(qsm + swz(row, col)) = v;
            }
            __syncwarp();
        }
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    };

    auto finish_item = [&]() {
        // full row sums across the quad
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        if (!rows_mode) {
            // merge the four warps' partial softmax states of the same 16 rows
            if (w > 0) {
                if (!mbar_wait(mempty, mphase ^ 1)) ok = false;
                float *mo = merge_o + (size_t)(w - 1) * 16 * D;
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    *(float2 *)(mo + qr * D + n * 8 + qc) = make_float2(o[n][0], o[n][1]);
                    *(float2 *)(mo + (qr + 8) * D + n * 8 + qc) = make_float2(o[n][2], o[n][3]);
                }
                if ((lane & 3) == 0) {
                    float *ml = merge_ml + (w - 1) * 32;
                    ml[qr] = m0;
                    ml[qr + 8] = m1;
                    ml[16 + qr] = l0;
                    ml[16 + qr + 8] = l1;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(mfull);
                mphase ^= 1;
                return;
            }
            if (!mbar_wait(mfull, mphase)) ok = false;
            float M0 = m0, M1 = m1;
#pragma unroll
            for (int k = 0; k < kConsumers - 1; ++k) {
                M0 = fmaxf(M0, merge_ml[k * 32 + qr]);
                M1 = fmaxf(M1, merge_ml[k * 32 + qr + 8]);
            }
            const float B0 = M0 == -INFINITY ? 0.f : M0, B1 = M1 == -INFINITY ? 0.f : M1;
            float w0 = fast_exp2(m0 - B0), w1 = fast_exp2(m1 - B1);
            l0 *= w0;
            l1 *= w1;
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                o[n][0] *= w0;
                o[n][1] *= w0;
                o[n][2] *= w1;
                o[n][3] *= w1;
            }
#pragma unroll
            for (int k = 0; k < kConsumers - 1; ++k) {
                const float *mo = merge_o + (size_t)k * 16 * D;
                const float e0 = fast_exp2(merge_ml[k * 32 + qr] - B0);
                const float e1 = fast_exp2(merge_ml[k * 32 + qr + 8] - B1);
                l0 += merge_ml[k * 32 + 16 + qr] * e0;
                l1 += merge_ml[k * 32 + 16 + qr + 8] * e1;
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    const float2 x0 = *(const float2 *)(mo + qr * D + n * 8 + qc);
                    const float2 x1 = *(const float2 *)(mo + (qr + 8) * D + n * 8 + qc);
                    o[n][0] += x0.x * e0;
                    o[n][1] += x0.y * e0;
                    o[n][2] += x1.x * e1;
                    o[n][3] += x1.y * e1;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(mempty);
            mphase ^= 1;
            m0 = M0;
            m1 = M1;
        }
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
        if (partial >= 0) {
            float *po = prm.partial_o + (size_t)partial * 16 * D;
            if (orow0 >= 0)
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *(float2 *)(po + qr * D + n * 8 + qc) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
            if (orow1 >= 0)
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *(float2 *)(po + (qr + 8) * D + n * 8 + qc) =
                        make_float2(o[n][2] * inv1, o[n][3] * inv1);
            if ((lane & 3) == 0) {
                float *pl = prm.partial_lse + (size_t)partial * 16;
                pl[qr] = l0 > 0.f ? m0 + __log2f(l0) : -INFINITY;
                pl[qr + 8] = l1 > 0.f ? m1 + __log2f(l1) : -INFINITY;
            }
        } else {
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
        }
    };

    auto compute_tile = [&](int kt, uint8_t *ks, uint8_t *vs) {
        const int valid = c - kt * kTile;  // tokens of this tile inside the context
        if (valid < kTile) {
            // tail tile: clear V rows past the context (stale or never-written slots)
            for (int ch = lane; ch < (kTile - valid) * (D / 8); ch += 32) {
                const int row = valid + ch / (D / 8), col = (ch % (D / 8)) * 8;
                *(uint4 *)(vs + swz(row, col)) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();
            __syncwarp();
        }
        const uint32_t ka = smem_u32(ks), va = smem_u32(vs), qa = smem_u32(qsm);
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
        if (mt.x < 0) {  // end marker: no more stages from this CTA's producer
            if (cur >= 0) finish_item();
            break;
        }
        if (mt.x != cur) {
            if (cur >= 0) finish_item();
            if (!ok) break;
            begin_item(mt.x);
            cur = mt.x;
        }
        const int kt = mt.y;
        const bool mine = rows_mode ? active : ((kt - kvb) % kConsumers) == w;
        if (mine && kt * kTile <= max_lim) {
            uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
            compute_tile(kt, ks, ks + 32 * D);
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
        record_error(prm.err, PK_ERR_TIMEOUT);
        *abort_flag = 1;
    }
}

// ---------------------------------------------------------------- split-K reduce
// out[row] = sum_p 2^(lse_p - M) o_p / sum_p 2^(lse_p - M), M = max_p lse_p
// (o_p already normalised by its own partition's sum; lse in the log2 domain).
template <int D>
__global__ void __launch_bounds__(128) reduce_kernel(const WsHeader *hdr, const ReduceItem *red,
                                                     const float *po, const float *plse,
                                                     const int32_t *ctx, const int32_t *qsl,
                                                     __nv_bfloat16 *out, int n_q_heads, int group) {
    const int n = hdr->n_reduce;
    for (int r = blockIdx.x; r < n; r += gridDim.x) {
        const ReduceItem it = red[r];
        const int qs0 = __ldg(qsl + it.seq);
        const int rows = (__ldg(qsl + it.seq + 1) - qs0) * group;
        for (int idx = threadIdx.x; idx < rows * (D / 4); idx += blockDim.x) {
            const int row = idx / (D / 4), c4 = idx % (D / 4);
            float M = -INFINITY;
            for (int p = 0; p < it.n_parts; ++p)
                M = fmaxf(M, plse[(size_t)(it.first_partial + p) * 16 + row]);
            float den = 0.f;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int p = 0; p < it.n_parts; ++p) {
                const float lse = plse[(size_t)(it.first_partial + p) * 16 + row];
                const float wgt = lse == -INFINITY ? 0.f : fast_exp2(lse - M);
                const float4 x =
                    *(const float4 *)(po + ((size_t)(it.first_partial + p) * 16 + row) * D + c4 * 4);
                den += wgt;
                acc.x += wgt * x.x;
                acc.y += wgt * x.y;
                acc.z += wgt * x.z;
                acc.w += wgt * x.w;
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            const int64_t orow = (int64_t)(qs0 + row / group) * n_q_heads + it.kvh * group + row % group;
            uint2 pk;
            pk.x = pack_bf16(acc.x * inv, acc.y * inv);
            pk.y = pack_bf16(acc.z * inv, acc.w * inv);
            *(uint2 *)(out + orow * D + c4 * 4) = pk;
        }
    }
}

WsLayout ws_layout(const pk_pool *p, int num_seqs, int num_tokens, int n_q_heads) {
    WsLayout L{};
    const int Hkv = p->n_kv_heads, g = n_q_heads / Hkv, D = p->head_dim;
    const int64_t row_groups = ((int64_t)num_tokens * g + kTile * kConsumers - 1) / (kTile * kConsumers);
    L.cap_rows = (int)(Hkv * (row_groups + num_seqs));
    L.cap_split = Hkv * num_seqs + p->tc_ctas * kItemsPerCta;
    L.cap_reduce = Hkv * num_seqs;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = up(sizeof(WsHeader));
    L.items_rows = off;
    off = up(off + (size_t)L.cap_rows * sizeof(WorkItem));
    L.items_split = off;
    off = up(off + (size_t)L.cap_split * sizeof(WorkItem));
    L.reduce = off;
    off = up(off + (size_t)L.cap_reduce * sizeof(ReduceItem));
    L.partial_o = off;
    off = up(off + (size_t)L.cap_split * 16 * D * sizeof(float));
    L.partial_lse = off;
    off = up(off + (size_t)L.cap_split * 16 * sizeof(float));
    L.total = off;
    return L;
}

template <int D>
int prepare(pk_pool *p) {
    const int smem = (int)smem_bytes<D>();
    cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "set attention smem size");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_tc_kernel<D>, kThreads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "attention occupancy");
    if (per_sm < 1) return fail(PK_ERR_UNSUPPORTED, "attention kernel does not fit on an SM");
    p->tc_ctas = per_sm * p->sm_count;
    return PK_OK;
}

template <int D>
int launch(const pk_pool *p, const AttnArgs &a, const WsLayout &L, cudaStream_t st) {
    uint8_t *ws = (uint8_t *)a.workspace;
    PlanArgs pa;
    pa.ctx = a.context_lens;
    pa.qsl = a.query_start_lens;
    pa.num_seqs = a.num_seqs;
    pa.num_tokens = a.num_tokens;
    pa.group = a.n_q_heads / p->n_kv_heads;
    pa.n_kv_heads = p->n_kv_heads;
    pa.block_size = p->block_size;
    pa.max_blocks = a.max_blocks_per_seq;
    pa.ncta = p->tc_ctas;
    pa.cap_rows = L.cap_rows;
    pa.cap_split = L.cap_split;
    pa.cap_reduce = L.cap_reduce;
    pa.hdr = (WsHeader *)ws;
    pa.items_rows = (WorkItem *)(ws + L.items_rows);
    pa.items_split = (WorkItem *)(ws + L.items_split);
    pa.reduce = (ReduceItem *)(ws + L.reduce);
    pa.err = p->d_err;
    plan_kernel<<<1, 1024, 0, st>>>(pa);

    TcParams tp;
    tp.q = (const __nv_bfloat16 *)a.q;
    tp.out = (__nv_bfloat16 *)a.out;
    tp.tables = a.block_tables;
    tp.ctx = a.context_lens;
    tp.qsl = a.query_start_lens;
    tp.max_blocks = a.max_blocks_per_seq;
    tp.n_q_heads = a.n_q_heads;
    tp.n_kv_heads = p->n_kv_heads;
    tp.group = pa.group;
    tp.block_size = p->block_size;
    tp.box_rows = p->block_size % kTile == 0 ? kTile : 8;
    tp.num_blocks = p->num_blocks;
    tp.scale_log2 = a.scale * 1.4426950408889634f;
    tp.hdr = pa.hdr;
    tp.items_rows = pa.items_rows;
    tp.items_split = pa.items_split;
    tp.partial_o = (float *)(ws + L.partial_o);
    tp.partial_lse = (float *)(ws + L.partial_lse);
    tp.err = p->d_err;
    attention_tc_kernel<D><<<p->tc_ctas, kThreads, smem_bytes<D>(), st>>>(p->tmap_k, p->tmap_v, tp);

    const int rgrid = std::max(1, std::min(L.cap_reduce, p->sm_count * 4));
    reduce_kernel<D><<<rgrid, 128, 0, st>>>(pa.hdr, pa.reduce, tp.partial_o, tp.partial_lse,
                                            a.context_lens, a.query_start_lens, tp.out,
                                            a.n_q_heads, pa.group);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "tensor-core attention launch");
}

}  // namespace

size_t tc_workspace_bytes(const pk_pool *p, int num_seqs, int num_tokens, int n_q_heads,
                          int /*max_blocks_per_seq*/) {
    return ws_layout(p, num_seqs, num_tokens, n_q_heads).total;
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
    const WsLayout L = ws_layout(p, a.num_seqs, a.num_tokens, a.n_q_heads);
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
