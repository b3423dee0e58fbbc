// Paged attention for causal prefill chunks on the fifth-generation tensor
// cores (tcgen05, accumulators in tensor memory): bf16 pools, head_dim 128,
// block_size a multiple of 16, groups g dividing 128.  Serves every sequence
// whose query rows (q_b tokens x g heads of a kv group) span more than one
// 16-row tile; decodes and chunks of a few tokens run in the decode kernel.
//
// What is computed ["Batching and PagedAttention", "Continuous batching":
// long prompts are split into chunks across steps; "PagedAttention & Continuous
// Batching" (study notes), "Block tables"]: query token i of a chunk of q
// tokens at context c sits at position c - q + i and attends to keys 0..c-q+i
// of its kv head, each key read through the sequence's block table.
//
// Structure.  A work item is 256 query rows (pairs (token, head of the
// group), token-major) of one (sequence, kv head), as two 128-row tiles; CTA i
// takes items i, i + gridDim.x, ...  Per 64-key stage:
//   - three producer warps load the stage's four 16-key blocks by TMA: K as two
//     2-D boxes per block (one per 64-column panel; warps 0 and 1) into the
//     canonical K-major 128-byte-swizzled layout [panel][64 keys][128 B], V as
//     one 3-D box per block [block][panel][16 keys][128 B] (warp 2).  K and V
//     have rings of their own: a K slot is refilled as soon as the stage's S
//     has completed, a V slot once its P V has, so each load is issued two to
//     three stages before it is read;
//   - one thread of the MMA warp issues, per row tile, S = Q K^T (M 128, N 64,
//     eight K-steps of 16) into one of two tensor-memory buffers, then, when
//     both tiles' softmax of the previous stage are done, O += P V (M 128,
//     N 128, four K-steps; V read MN-major);
//   - per row tile, four softmax warps own one query row per thread (two
//     warpgroups share each SM sub-partition and hide each other's latency):
//     they read the row of S
//     from tensor memory (no shuffles), mask causally, keep the running max m
//     and sum l in fp32 (the reference m moves, and O is rescaled in tensor
//     memory, only when a score exceeds it by more than 2^8), and write P as
//     bf16 into a 128-byte-swizzled shared buffer, the A operand of P V.
// Every wait is bounded (2 s); on expiry the kernel records PK_ERR_TIMEOUT,
// each warp waits (bounded) for its own copies and tensor-core work, and the
// CTA releases its tensor memory and returns.  Block ids are range-checked.
#include "tc_common.cuh"

#include <algorithm>
#include <cstdlib>

namespace pk {
namespace {

using namespace tc;

constexpr int kUD = 128;                // head dim
constexpr int kURows = 128;             // query rows per row tile (UMMA M)
constexpr int kUTiles = 2;              // row tiles per item: 256 query rows share each KV stage
constexpr int kUItemRows = kURows * kUTiles;
constexpr int kUKeys = 64;              // keys per stage
constexpr int kUKStages = 4;            // K ring: a slot is free once the stage's S = Q K^T has completed
constexpr int kUVStages = 3;            // V ring: a slot is free once the stage's O += P V has completed
constexpr int kUMma = 8;                // warp 8: tensor memory and MMA issue
constexpr int kUProd0 = 9;              // warps 9, 10: K panel 0, 1; warp 11: V
constexpr int kUThreads = 12 * 32;      // warps 0..3 and 4..7: softmax of row tile 0 and 1
constexpr uint32_t kUTmemCols = 512;    // S[t][b] at 128 t + 64 b, O[t] at 256 + 128 t
constexpr float kURescaleLog2 = 8.f;

constexpr uint32_t kUQBytes = kURows * kUD * 2;       // per tile: [panel][128 rows][128 B]
constexpr uint32_t kUKBytes = kUKeys * kUD * 2;       // [panel][64 keys][128 B]
constexpr uint32_t kUVBytes = kUKeys * kUD * 2;       // [block][panel][16 keys][128 B]
constexpr uint32_t kUPBytes = kURows * kUKeys * 2;    // per tile: [128 rows][128 B]
constexpr uint32_t kUOffQ = 0;
constexpr uint32_t kUOffK = kUOffQ + kUTiles * kUQBytes;
constexpr uint32_t kUOffV = kUOffK + kUKStages * kUKBytes;
constexpr uint32_t kUOffP = kUOffV + kUVStages * kUVBytes;
constexpr uint32_t kUOffPlan = kUOffP + kUTiles * kUPBytes;
constexpr uint32_t kUOffBar = kUOffPlan + (3 * kPlanLen * 4 + 15) / 16 * 16;
// barriers: k_full[K slot], k_empty[K slot], v_full[V slot], v_empty[V slot]; per
// row tile: s_full[2], s_free[2], p_full, pv_done, q_full, o_full, o_free; mma_done
constexpr uint32_t kUPerTileBars = 9;
constexpr uint32_t kUNumBars = 2 * kUKStages + 2 * kUVStages + kUTiles * kUPerTileBars + 1;
constexpr uint32_t kUOffMisc = kUOffBar + kUNumBars * 8;  // tensor memory address, abort flag
constexpr uint32_t kUSmem = kUOffMisc + 16 + 1024;        // + alignment slack
static_assert(kUSmem <= 227 * 1024 - 64, "chunk kernel shared memory");

// instruction descriptors (kind::f16): fp32 accumulate, bf16 A and B, M = 128
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);  // B MN-major

// Shared-memory matrix descriptor: 128-byte swizzle, byte offsets lbo / sbo.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version of sm_100
    d |= (uint64_t)2 << 61;  // 128-byte swizzle
    return d;
}
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
                 :
                 : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                 : "memory");
}
struct UParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables, *ctx, *qsl;
    int seq0, nseq, max_blocks, n_q_heads, n_kv_heads, group, block_size, num_blocks, num_tokens;
    float scale_log2;
    int *err;
};

struct UItem {
    int b, kvh, rt, c, qn, qs0, rows, nkt;
};

// Per-row-tile barriers.
struct UTileBars {
    uint64_t *s_full, *s_free, *p_full, *pv_done, *q_full, *o_full, *o_free;
};

__global__ void __launch_bounds__(kUThreads, 1)
attention_chunk_umma_kernel(const __grid_constant__ CUtensorMap tmk2,  // K: 2-D, 16-row boxes
                            const __grid_constant__ CUtensorMap tmv3,  // V: 3-D, 16 rows x 2 panels
                            const UParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = prm.group, Hq = prm.n_q_heads, Hkv = prm.n_kv_heads, bs = prm.block_size;
    const int nseq = prm.nseq;
    int *item_pre = (int *)(sm + kUOffPlan);
    int *s_qsl = item_pre + kPlanLen;
    int *s_ctx = s_qsl + kPlanLen;
    uint64_t *k_full = (uint64_t *)(sm + kUOffBar);
    uint64_t *k_empty = k_full + kUKStages;
    uint64_t *v_full = k_empty + kUKStages;
    uint64_t *v_empty = v_full + kUVStages;
    uint64_t *tile_bars = v_empty + kUVStages;
    uint64_t *mma_done = tile_bars + kUTiles * kUPerTileBars;
    auto tb = [&](int t) {
        uint64_t *q = tile_bars + t * kUPerTileBars;
        return UTileBars{q, q + 2, q + 4, q + 5, q + 6, q + 7, q + 8};
    };
    uint32_t *tmem_slot = (uint32_t *)(sm + kUOffMisc);
    volatile int *abort_flag = (volatile int *)(sm + kUOffMisc + 4);
    __shared__ int s_nitems;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kUKStages; ++s) {
            mbar_init(&k_full[s], 2);  // both K producers
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kUVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int t = 0; t < kUTiles; ++t) {
            const UTileBars B = tb(t);
            for (int b = 0; b < 2; ++b) {
                mbar_init(&B.s_full[b], 1);
                mbar_init(&B.s_free[b], 4);
            }
            mbar_init(B.p_full, 4);
            mbar_init(B.pv_done, 1);
            mbar_init(B.q_full, 4);
            mbar_init(B.o_full, 1);
            mbar_init(B.o_free, 4);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kUMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kUTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == kUProd0) {
        // items: every sequence whose rows need more than one 16-row tile
        // contributes ceil(rows / 256) items per kv head
        int run = 0;
        for (int base = 0; base < nseq; base += 32) {
            const int i = base + lane;
            int n = 0;
            if (i < nseq) {
                const int b = prm.seq0 + i;
                const int s0 = __ldg(prm.qsl + b), s1 = __ldg(prm.qsl + b + 1), c = __ldg(prm.ctx + b);
                s_qsl[i] = s0;
                s_ctx[i] = c;
                if (i == nseq - 1) s_qsl[nseq] = s1;
                const int qn = s1 - s0;
                const bool ok = s0 >= 0 && s1 <= prm.num_tokens && qn >= 1 && c >= qn &&
                                (long long)(c + bs - 1) / bs <= prm.max_blocks;
                if (ok && qn * g > kTile) n = (qn * g + kUItemRows - 1) / kUItemRows * Hkv;
            }
            int inc = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            if (i < nseq) item_pre[i + 1] = run + inc;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) {
            item_pre[0] = 0;
            s_nitems = run;
        }
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = s_nitems;

    auto item_of = [&](int idx, UItem &it) {
        const int b = find_seq(item_pre, nseq, idx);
        const int local = idx - item_pre[b];
        it.b = b;
        it.qs0 = s_qsl[b];
        it.qn = s_qsl[b + 1] - it.qs0;
        it.c = s_ctx[b];
        it.rows = it.qn * g;
        const int nit = (it.rows + kUItemRows - 1) / kUItemRows;
        it.kvh = local / nit;
        it.rt = local - it.kvh * nit;
        const int last_row = min((it.rt + 1) * kUItemRows, it.rows) - 1;
        it.nkt = (it.c - it.qn + last_row / g) / kUKeys + 1;
    };

    if (warp >= kUProd0) {
        // ------------------------------------------------------------ producers
        // warps 9 and 10: K panel 0 and 1 of the stage's four 16-key blocks into
        // [panel][64 keys][128 B]; warp 11: V, one 3-D box per block into
        // [block][panel][16 keys][128 B]
        const int p = warp - kUProd0;
        const bool is_v = p == 2;
        const int nst = is_v ? kUVStages : kUKStages;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        if (lane == 0) prefetch_tmap(is_v ? &tmv3 : &tmk2);
        int n = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x) {
            UItem it;
            item_of(idx, it);
            const int32_t *table = prm.tables + (long long)(prm.seq0 + it.b) * prm.max_blocks;
            const int nblk = (it.c + bs - 1) / bs;
            int base = 0;
            int cur = lane < nblk ? __ldg(table + lane) : 0;
            int nxt = 32 + lane < nblk ? __ldg(table + 32 + lane) : 0;
            for (int j = 0; j < it.nkt; ++j, ++n) {
                const int s = n % nst;
                if (n >= nst && !mbar_wait(&empty[s], (uint32_t)(n / nst - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (*abort_flag) {
                    ok = false;
                    break;
                }
                int ys[4];
#pragma unroll
                for (int jb = 0; jb < 4; ++jb) {
                    const int k0 = j * kUKeys + jb * kTile;
                    ys[jb] = -1;
                    if (k0 < it.c) {  // warp-uniform
                        const int blk = k0 / bs;
                        while (blk >= base + 32) {
                            base += 32;
                            cur = nxt;
                            nxt = base + 32 + lane < nblk ? __ldg(table + base + 32 + lane) : 0;
                        }
                        int phys = __shfl_sync(0xffffffffu, cur, blk - base);
                        if (phys < 0 || phys >= prm.num_blocks) {
                            if (lane == 0) record_error(prm.err, PK_ERR_BAD_INDEX);
                            phys = 0;
                        }
                        ys[jb] = (phys * Hkv + it.kvh) * bs + k0 % bs;
                    }
                }
                if (lane == 0) {
                    uint32_t bytes = 0;
#pragma unroll
                    for (int jb = 0; jb < 4; ++jb)
                        if (ys[jb] >= 0) bytes += is_v ? 4096u : 2048u;
                    if (bytes == 0) {
                        mbar_arrive(&full[s]);  // keys past the context: nothing to load
                    } else {
                        mbar_arrive_expect_tx(&full[s], bytes);
                        uint8_t *dst = is_v ? sm + kUOffV + (size_t)s * kUVBytes
                                            : sm + kUOffK + (size_t)s * kUKBytes + p * 8192;
#pragma unroll
                        for (int jb = 0; jb < 4; ++jb) {
                            if (ys[jb] < 0) continue;
                            if (is_v) tma_load_3d(dst + jb * 4096, &tmv3, 0, ys[jb], 0, &full[s]);
                            else tma_load_2d(dst + jb * 2048, &tmk2, p * 64, ys[jb], &full[s]);
                        }
                    }
                }
                __syncwarp();
            }
        }
        if (!ok) {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
        // never leave with a copy still writing into this CTA's shared memory
        for (int m = max(0, n - nst); m < n; ++m) mbar_wait(&full[m % nst], (uint32_t)(m / nst) & 1);
    } else if (warp < kUMma) {
        // ------------------------------------------------------------ softmax + epilogue
        const int t = warp >> 2;             // row tile of this warpgroup
        const int sp = warp & 3;             // tensor-memory lane quarter of this warp
        const int r = sp * 32 + lane;        // the query row this thread owns
        const UTileBars B = tb(t);
        const uint32_t row_t = tmem + ((uint32_t)(sp * 32) << 16);
        const uint32_t s_col = (uint32_t)(t * 128), o_col = (uint32_t)(256 + t * 128);
        uint8_t *qbuf = sm + kUOffQ + t * kUQBytes;
        uint8_t *pbuf = sm + kUOffP + t * kUPBytes + r * 128;
        int n = 0, n_item = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x, ++n_item) {
            UItem it;
            item_of(idx, it);
            const int R = it.rt * kUItemRows + t * kURows + r;
            const bool valid = R < it.rows;
            const int tok = valid ? R / g : 0, hh = valid ? R % g : 0;
            const int pos = it.c - it.qn + tok;
            const long long qrow = ((long long)(it.qs0 + tok) * Hq + it.kvh * g + hh) * kUD;
            // Q row into the K-major 128-byte-swizzled layout (the previous item's
            // MMAs have completed: its o_full was seen)
            {
                const uint4 *src = (const uint4 *)(prm.q + qrow);
#pragma unroll
                for (int ch = 0; ch < 16; ++ch) {
                    const uint4 v = valid ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
                    const int pn = ch >> 3, c8 = ch & 7;
                    *(uint4 *)(qbuf + pn * (kURows * 128) + r * 128 + ((c8 ^ (r & 7)) << 4)) = v;
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(B.q_full);
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < it.nkt; ++j, ++n) {
                const int b = n & 1;
                if (!mbar_wait(&B.s_full[b], (uint32_t)(n >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_after();
                uint32_t sv[64];
                tmem_ld64(row_t + s_col + (uint32_t)(b * 64), sv);
                tmem_wait_ld();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B.s_free[b]);
                const int k0 = j * kUKeys;
                // scores in log2 units are s * scale_log2; the running max is kept in
                // those units, the raw max (scale > 0) is taken first.  Stages wholly
                // below every row's diagonal skip the mask.
                float mx = -INFINITY;
                if (__all_sync(0xffffffffu, valid && k0 + kUKeys - 1 <= pos)) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
                } else {
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        const float sc = (valid && k0 + i <= pos) ? __uint_as_float(sv[i]) : -INFINITY;
                        sv[i] = __float_as_uint(sc);
                        mx = fmaxf(mx, sc);
                    }
                }
                mx *= prm.scale_log2;
                // the P V of the previous stage has finished: P is free and O is final
                if (n >= 1 && !mbar_wait(B.pv_done, (uint32_t)(n - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (__any_sync(0xffffffffu, mx > m + kURescaleLog2)) {
                    const float mn = fmaxf(m, mx);
                    const float alpha = mn == -INFINITY ? 1.f : fast_exp2(m - mn);
                    if (j > 0) {  // O holds earlier stages: rescale it in place
                        tc_after();
#pragma unroll 1
                        for (int q8 = 0; q8 < 8; ++q8) {
                            uint32_t ov[16];
                            tmem_ld16(row_t + o_col + (uint32_t)(q8 * 16), ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                            tmem_st16(row_t + o_col + (uint32_t)(q8 * 16), ov);
                        }
                        tmem_wait_st();
                    }
                    m = mn;
                    l *= alpha;
                }
                const float bm = m == -INFINITY ? 0.f : m;
                const float sl = prm.scale_log2;
                float ps = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    float pv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        pv[i] = fast_exp2(fmaf(__uint_as_float(sv[8 * c8 + i]), sl, -bm));
                        ps += pv[i];
                    }
                    uint4 w;
                    w.x = pack_bf16(pv[0], pv[1]);
                    w.y = pack_bf16(pv[2], pv[3]);
                    w.z = pack_bf16(pv[4], pv[5]);
                    w.w = pack_bf16(pv[6], pv[7]);
                    *(uint4 *)(pbuf + ((c8 ^ (r & 7)) << 4)) = w;
                }
                l += ps;
                const int valid_keys = it.c - k0;
                if (valid_keys < kUKeys) {
                    // V rows past the context (stale or unloaded) must be zero: P is 0
                    // there.  Both warpgroups write the same zeros, after the stage's V
                    // has landed; the MMA thread waits for both before either P V.
                    if (!mbar_wait(&v_full[n % kUVStages], (uint32_t)(n / kUVStages) & 1)) {
                        ok = false;
                        break;
                    }
                    uint8_t *vs = sm + kUOffV + (size_t)(n % kUVStages) * kUVBytes;
                    for (int i = r; i < (kUKeys - valid_keys) * 16; i += kURows) {
                        const int key = valid_keys + i / 16, ch = i % 16;
                        *(uint4 *)(vs + (key >> 4) * 4096 + (ch >> 3) * 2048 + (key & 15) * 128 + (ch & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                fence_proxy_async();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(B.p_full);
            }
            if (!ok) break;
            // epilogue: O / l for this thread's row
            if (!mbar_wait(B.o_full, (uint32_t)n_item & 1)) {
                ok = false;
                break;
            }
            tc_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *dst = (uint4 *)(prm.out + qrow);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint32_t ov[32];
                tmem_ld32(row_t + o_col + (uint32_t)(q4 * 32), ov);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(ov[8 * c8 + 0]) * inv, __uint_as_float(ov[8 * c8 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(ov[8 * c8 + 2]) * inv, __uint_as_float(ov[8 * c8 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(ov[8 * c8 + 4]) * inv, __uint_as_float(ov[8 * c8 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(ov[8 * c8 + 6]) * inv, __uint_as_float(ov[8 * c8 + 7]) * inv);
                        dst[q4 * 4 + c8] = w;
                    }
                }
            }
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(B.o_free);
        }
        if (!ok) {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else {
        // ------------------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
            bool ok = true;
            int n = 0, n_item = 0;
            // O += P V of stage nn for both row tiles (both softmax warpgroups done)
            auto pv = [&](int nn, bool first) -> bool {
                for (int t = 0; t < kUTiles; ++t) {
                    const UTileBars B = tb(t);
                    if (!mbar_wait(B.p_full, (uint32_t)nn & 1)) return false;
                    if (first && n_item > 0 && !mbar_wait(B.o_free, (uint32_t)(n_item - 1) & 1)) return false;
                }
                const int s = nn % kUVStages;
                if (!mbar_wait(&v_full[s], (uint32_t)(nn / kUVStages) & 1)) return false;
                tc_after();
                const uint32_t va = smem_u32(sm + kUOffV + (size_t)s * kUVBytes);
                for (int t = 0; t < kUTiles; ++t) {
                    const uint32_t pa = smem_u32(sm + kUOffP + t * kUPBytes);
#pragma unroll
                    for (int kp = 0; kp < 4; ++kp)
                        umma_f16(tmem + 256u + (uint32_t)(t * 128), sdesc(pa + kp * 32, 16, 1024),
                                 sdesc(va + kp * 4096, 2048, 1024), kIdescPV, (first && kp == 0) ? 0u : 1u);
                    umma_commit(tb(t).pv_done);
                }
                umma_commit(&v_empty[s]);
                return true;
            };
            for (int idx = blockIdx.x; ok && idx < n_items; idx += gridDim.x, ++n_item) {
                UItem it;
                item_of(idx, it);
                for (int t = 0; t < kUTiles && ok; ++t) ok = mbar_wait(tb(t).q_full, (uint32_t)n_item & 1);
                if (!ok) break;
                tc_after();
                for (int j = 0; j < it.nkt; ++j, ++n) {
                    const int s = n % kUKStages, b = n & 1;
                    bool got = mbar_wait(&k_full[s], (uint32_t)(n / kUKStages) & 1);
                    for (int t = 0; t < kUTiles && got; ++t)
                        if (n >= 2) got = mbar_wait(&tb(t).s_free[b], (uint32_t)((n >> 1) - 1) & 1);
                    if (!got || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t ka = smem_u32(sm + kUOffK + (size_t)s * kUKBytes);
                    for (int t = 0; t < kUTiles; ++t) {
                        const uint32_t qa = smem_u32(sm + kUOffQ + t * kUQBytes);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_f16(tmem + (uint32_t)(t * 128 + b * 64),
                                     sdesc(qa + (kk >> 2) * (kURows * 128) + (kk & 3) * 32, 16, 1024),
                                     sdesc(ka + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), kIdescS,
                                     kk > 0 ? 1u : 0u);
                        umma_commit(&tb(t).s_full[b]);
                    }
                    umma_commit(&k_empty[s]);  // the K slot is free once both S have completed
                    if (j > 0 && !pv(n - 1, j == 1)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                if (!pv(n - 1, it.nkt == 1)) {
                    ok = false;
                    break;
                }
                for (int t = 0; t < kUTiles; ++t) umma_commit(tb(t).o_full);
            }
            if (!ok) {
                record_error(prm.err, PK_ERR_TIMEOUT);
                *abort_flag = 1;
            }
            // all tensor-core work of this CTA has completed before its memory is freed
            umma_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
        __syncwarp();
    }
    tc_before();
    __syncthreads();
    if (warp == kUMma) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols)
                     : "memory");
    }
}

}  // namespace

// Serves bf16 pools with head_dim 128 and 16-row tile boxes (block_size a
// multiple of 16), and groups dividing 128; PK_CHUNK_MMA_SYNC=1 selects the
// mma.sync chunk kernel instead.
int chunk_umma_prepare_pool(pk_pool *p) {
    p->umma_ok = false;
    const char *e = getenv("PK_CHUNK_MMA_SYNC");
    if (p->head_dim != kUD || !p->tile_map3d || (e && e[0] == '1')) return PK_OK;
    cudaError_t ce = cudaFuncSetAttribute(attention_chunk_umma_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kUSmem);
    if (ce != cudaSuccess) return cuda_fail(ce, "set chunk (tcgen05) smem size");
    int rc = encode_pool_map(&p->tmap_k2, p->k_base, p, kTile);
    if (rc == PK_OK) rc = encode_pool_map(&p->tmap_v2, p->v_base, p, kTile);
    if (rc != PK_OK) return rc;
    p->umma_ok = true;
    return PK_OK;
}

bool chunk_umma_applies(const pk_pool *p, const AttnArgs &a) {
    const int g = a.n_q_heads / p->n_kv_heads;
    return p->umma_ok && g >= 1 && kURows % g == 0;
}

int launch_chunk_umma(const pk_pool *p, const AttnArgs &a, cudaStream_t st) {
    UParams u;
    u.q = (const __nv_bfloat16 *)a.q;
    u.out = (__nv_bfloat16 *)a.out;
    u.tables = a.block_tables;
    u.ctx = a.context_lens;
    u.qsl = a.query_start_lens;
    u.max_blocks = a.max_blocks_per_seq;
    u.n_q_heads = a.n_q_heads;
    u.n_kv_heads = p->n_kv_heads;
    u.group = a.n_q_heads / p->n_kv_heads;
    u.block_size = p->block_size;
    u.num_blocks = p->num_blocks;
    u.num_tokens = a.num_tokens;
    u.scale_log2 = a.scale * 1.4426950408889634f;
    u.err = p->d_err;
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        u.seq0 = s0;
        u.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        attention_chunk_umma_kernel<<<p->sm_count, kUThreads, kUSmem, st>>>(p->tmap_k2, p->tmap_v, u);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "chunk attention (tcgen05) launch");
}

}  // namespace pk
