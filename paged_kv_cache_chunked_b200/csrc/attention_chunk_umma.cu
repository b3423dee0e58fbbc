// Paged attention for causal prefill chunks on the fifth-generation tensor
// cores (tcgen05, operands and accumulators in tensor memory): bf16 pools,
// head_dim 64 or 128, block_size a multiple of 16, groups g dividing 128.  Serves
// every sequence of two or more query tokens when the block-streaming decode
// kernel takes the one-token rows of the batch (groups of at most 8), else
// every sequence whose query rows (q_b tokens x g heads of a kv group) span more
// than one 16-row tile, the rest running in the tile-streaming decode kernel.
//
// What is computed ["Batching and PagedAttention", "Continuous batching":
// long prompts are split into chunks across steps; "PagedAttention & Continuous
// Batching" (study notes), "Block tables"]: query token i of a chunk of q
// tokens at context c sits at position c - q + i and attends to keys 0..c-q+i
// of its kv head, each key read through the sequence's block table.
//
// Structure.  A work item is 256 query rows (pairs (token, head of the
// group), token-major) of one (sequence, kv head), as two 128-row tiles; the
// CTAs take the items sequence by sequence, heaviest sequence first, in the
// snake order of umma_common.cuh.  Per 128-key stage:
//   - producer warps load the stage's eight 16-key blocks by TMA: K as one
//     2-D box per block and 64-column panel (warp 9 panel 0, warp 10 panel 1
//     at head dim 128) into the canonical K-major 128-byte-swizzled layout
//     [panel][128 keys][128 B], V as one 3-D box per block [block][panel][16
//     keys][128 B] (warp 11).  Lane j of a producer looks up and issues block j, so a
//     stage's eight table lookups and boxes go out together.  K and V have
//     rings of their own: a K slot is refilled once the stage's S has
//     completed, a V slot once its P V has.  On a stage that runs past the
//     context the V warp zeroes the rows past it (P is 0 there, the stale rows
//     may hold anything) before it releases the stage;
//   - one thread of the MMA warp issues, per row tile t, O_t += P_t V of the
//     previous stage (A = P_t read from tensor memory, B = V MN-major; M 128,
//     N = head dim, eight K-steps) and then S_t = Q_t K^T of this stage (M 128,
//     N 128, head dim / 16 K-steps) into the same tensor-memory columns: the tensor core runs
//     one thread's MMAs in order, so S_t overwrites P_t only after P_t V has
//     read it.  Tile 1's MMAs run while tile 0's softmax works and the other
//     way round;
//   - per row tile, four softmax warps own one query row per thread: they read
//     the row of S from tensor memory, mask causally, keep the running max m and
//     sum l in fp32 (the reference m moves, and O is rescaled in tensor memory,
//     only when a score exceeds it by more than 2^8), and write P as packed bf16
//     over the first 64 columns of S.  When S_t of a stage is complete, P_t V of
//     the previous stage is too (its commit covers every earlier MMA), so O_t is
//     stable for the whole softmax.
// Each tcgen05.mma has an issue cost of its own, so the stage is 128 keys wide:
// S MMAs with N = 128 do twice the work per instruction of N = 64 ones.
// Every wait is bounded (2 s); on expiry the kernel records PK_ERR_TIMEOUT,
// each warp waits (bounded) for its own copies and tensor-core work, and the
// CTA releases its tensor memory and returns.  Block ids are range-checked.
#include "umma_common.cuh"

#include <algorithm>
#include <cstdlib>

namespace pk {
namespace {

using namespace tc;

constexpr int kURows = 128;             // query rows per row tile (UMMA M)
constexpr int kUTiles = 2;              // row tiles per item: 256 query rows share each KV stage
constexpr int kUItemRows = kURows * kUTiles;
constexpr int kUKeys = 128;             // keys per stage (UMMA N of S)
constexpr int kUBlk = kUKeys / 16;      // 16-key blocks per stage
constexpr int kUKStages = 2;            // K ring: a slot is free once the stage's S = Q K^T has completed
constexpr int kUVStages = 2;            // V ring: a slot is free once the stage's O += P V has completed
constexpr int kUMma = 8;                // warp 8: tensor memory and MMA issue
constexpr int kUProd0 = 9;              // warps 9, 10: K panel 0, 1 (head dim 64: warp 9 only); warp 11: V
constexpr int kUThreads = 12 * 32;      // warps 0..3 and 4..7: softmax of row tile 0 and 1
constexpr uint32_t kUTmemCols = 512;    // S[t] (P[t] over its first 64 columns) at 128 t, O[t] at 256 + 128 t
constexpr float kURescaleLog2 = 8.f;
// Register split: the kernel launches with kURegLaunch registers a thread; the
// two softmax warpgroups then take kURegSoftmax and the MMA / producer warpgroup
// keeps kURegOther.  The split uses exactly the launch's registers (setmaxnreg
// can only hand out what the block was launched with), and the host checks the
// compiled register count before it enables this kernel.
constexpr int kURegLaunch = 168, kURegSoftmax = 176, kURegOther = 152;
static_assert(256 * kURegSoftmax + 128 * kURegOther <= kUThreads * kURegLaunch, "register split");

// Shared-memory layout and instruction descriptors for head dim D (64 or 128).
template <int D>
struct UGeo {
    static constexpr int kPanels = D / 64;                    // 64-column (128-byte) panels
    static constexpr uint32_t QBytes = kURows * D * 2;        // per tile: [panel][128 rows][128 B]
    static constexpr uint32_t KBytes = kUKeys * D * 2;        // [panel][128 keys][128 B]
    static constexpr uint32_t KPanel = kUKeys * 128;          // bytes of one K panel
    static constexpr uint32_t VBlock = 16 * D * 2;            // one 16-key block of V: [panel][16 keys][128 B]
    static constexpr uint32_t VBytes = kUKeys * D * 2;        // [block][panel][16 keys][128 B]
    static constexpr uint32_t OffQ = 0;
    static constexpr uint32_t OffK = OffQ + kUTiles * QBytes;
    static constexpr uint32_t OffV = OffK + kUKStages * KBytes;
    static constexpr uint32_t OffPlan = OffV + kUVStages * VBytes;
    static constexpr uint32_t OffBar = OffPlan + ((3 * kPlanLen + kOrderInts) * 4 + 15) / 16 * 16;
    // barriers: k_full[K slot], k_empty[K slot], v_full[V slot], v_empty[V slot],
    // v_tma; per row tile: s_full, p_full, q_full, o_full, o_free; mma_done
    static constexpr uint32_t PerTileBars = 5;
    static constexpr uint32_t NumBars = 2 * kUKStages + 2 * kUVStages + 1 + kUTiles * PerTileBars + 1;
    static constexpr uint32_t OffMisc = OffBar + NumBars * 8;  // tensor memory address, abort flag
    static constexpr uint32_t Smem = OffMisc + 16 + 1024;      // + alignment slack
    static_assert(Smem <= 227 * 1024 - 64, "chunk kernel shared memory");
    // O += P V (kind::f16): fp32 accumulate, bf16 A and B, B MN-major, M = 128, N = D
    static constexpr uint32_t IdescPV =
        (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | (((uint32_t)D >> 3) << 17) | ((128u >> 4) << 24);
};
constexpr uint32_t kUPerTileBars = 5;
// S = Q K^T (kind::f16): fp32 accumulate, bf16 A and B, M = 128, N = 128 keys
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct UParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables, *ctx, *qsl;
    int seq0, nseq, max_blocks, n_q_heads, n_kv_heads, group, block_size, num_blocks, num_tokens;
    int min_rows;  // a sequence is served when its query rows (tokens x group heads) exceed this
    float scale_log2;
    int *err;
};

struct UItem {
    int b, kvh, rt, c, qn, qs0, rows, nkt;
};

// Per-row-tile barriers.
struct UTileBars {
    uint64_t *s_full, *p_full, *q_full, *o_full, *o_free;
};

template <int D>
__global__ void __launch_bounds__(kUThreads, 1)
attention_chunk_umma_kernel(const __grid_constant__ CUtensorMap tmk2,  // K: 2-D, 16-row boxes
                            const __grid_constant__ CUtensorMap tmv3,  // V: 3-D, 16 rows x 2 panels
                            const UParams prm) {
    using G = UGeo<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = prm.group, Hq = prm.n_q_heads, Hkv = prm.n_kv_heads, bs = prm.block_size;
    const int nseq = prm.nseq;
    int *grp_pre = (int *)(sm + G::OffPlan);  // groups (256-row blocks) of sequences 0..i-1
    int *s_qsl = grp_pre + kPlanLen;
    int *s_ctx = s_qsl + kPlanLen;
    const ChunkOrder order(s_ctx + kPlanLen);
    uint64_t *k_full = (uint64_t *)(sm + G::OffBar);
    uint64_t *k_empty = k_full + kUKStages;
    uint64_t *v_full = k_empty + kUKStages;
    uint64_t *v_empty = v_full + kUVStages;
    uint64_t *v_tma = v_empty + kUVStages;  // V of a stage that runs past the context
    uint64_t *tile_bars = v_tma + 1;
    uint64_t *mma_done = tile_bars + kUTiles * kUPerTileBars;
    auto tb = [&](int t) {
        uint64_t *q = tile_bars + t * kUPerTileBars;
        return UTileBars{q, q + 1, q + 2, q + 3, q + 4};
    };
    uint32_t *tmem_slot = (uint32_t *)(sm + G::OffMisc);
    volatile int *abort_flag = (volatile int *)(sm + G::OffMisc + 4);
    __shared__ int s_ngroups, s_nchunk;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kUKStages; ++s) {
            mbar_init(&k_full[s], G::kPanels);  // one K producer per panel
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < kUVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(v_tma, 1);
        for (int t = 0; t < kUTiles; ++t) {
            const UTileBars B = tb(t);
            mbar_init(B.s_full, 1);
            mbar_init(B.p_full, 4);
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
        // groups: every sequence whose rows need more than one 16-row tile
        // contributes ceil(rows / 256) groups, each of Hkv items (one per kv head)
        int run = 0, nchunk = 0;
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
                if (ok && qn * g > prm.min_rows) n = (qn * g + kUItemRows - 1) / kUItemRows;
            }
            int inc = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            if (i < nseq) grp_pre[i + 1] = run + inc;
            run += __shfl_sync(0xffffffffu, inc, 31);
            // the chunk sequences, in window order, for the ranking
            const unsigned has = __ballot_sync(0xffffffffu, n > 0);
            const int pos = nchunk + __popc(has & ((1u << lane) - 1));
            if (n > 0 && pos < kRankCap) order.cseq[pos] = i;
            nchunk += __popc(has);
        }
        if (lane == 0) {
            grp_pre[0] = 0;
            s_ngroups = run;
            s_nchunk = nchunk;
        }
    }
    __syncthreads();
    const int n_groups = s_ngroups;
    const int n_items = n_groups * Hkv;
    if (s_nchunk <= kRankCap)
        rank_chunk_seqs<kUItemRows, kUKeys>(order, s_nchunk, grp_pre, s_qsl, s_ctx, g, Hkv, threadIdx.x, kUThreads);
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;
    // Launched as a programmatic dependent of the kernel before it on the stream:
    // the plan above reads only the query offsets and lengths, which no kernel
    // of the call writes; the pool, the queries, the tables and the output are
    // touched only after this wait, which also covers every kernel before that
    // one.  Dependents are signalled after the wait, so a kernel launched behind
    // this one (the decode rows of a mixed step) may start work at once: the
    // step's rows and everything before this kernel are complete by then.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp < kUMma) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kURegSoftmax));
    else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kURegOther));

    // the item at position idx of the ranked list (the chunk-sequence count is
    // read back from shared memory: kept in a register across the item loops it
    // would cost the softmax warps a register)
    auto item_of = [&](int idx, UItem &it) {
        int local;
        ranked_item(order, s_nchunk, grp_pre, nseq, Hkv, idx, it.b, local);
        const int nit = grp_pre[it.b + 1] - grp_pre[it.b];
        it.kvh = local / nit;
        it.rt = local - it.kvh * nit;
        it.qs0 = s_qsl[it.b];
        it.qn = s_qsl[it.b + 1] - it.qs0;
        it.c = s_ctx[it.b];
        it.rows = it.qn * g;
        it.nkt = block_stages<kUItemRows, kUKeys>(it.c, it.qn, g, it.rt);
    };

    if (warp >= kUProd0) {
        // ------------------------------------------------------------ producers
        // warps 9 and 10: K panel 0 and 1 of the stage's eight 16-key blocks into
        // [panel][128 keys][128 B]; warp 11: V, one 3-D box per block into
        // [block][panel][16 keys][128 B]
        const int p = warp - kUProd0;
        const bool is_v = p == 2;
        const bool active = is_v || p < G::kPanels;  // head dim 64: one K panel, warp 10 idles
        const int nst = is_v ? kUVStages : kUKStages;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        if (lane == 0) prefetch_tmap(is_v ? &tmv3 : &tmk2);
        int n = 0, ntail = 0;
        bool ok = true;
        for (int idx = blockIdx.x; active && ok && idx < n_items;
             idx = snake_next(idx, blockIdx.x, gridDim.x)) {
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
                // lane jb (< 8) looks up 16-key block jb of the stage: one division
                // per lane, all lanes at once.  The table window advances once a
                // stage, to the stage's first block; a stage spans at most 8 blocks,
                // so all of them lie in cur (base..) or nxt (base + 32..)
                const int blk0 = j * kUKeys / bs;  // warp-uniform
                while (blk0 >= base + 32) {
                    base += 32;
                    cur = nxt;
                    nxt = base + 32 + lane < nblk ? __ldg(table + base + 32 + lane) : 0;
                }
                const int k0 = j * kUKeys + lane * kTile;
                const bool has = lane < kUBlk && k0 < it.c;
                const int blk = has ? k0 / bs : blk0;
                const int idx = blk - base;        // 0 .. 39
                const int pa = __shfl_sync(0xffffffffu, cur, idx & 31);
                const int pb = __shfl_sync(0xffffffffu, nxt, idx & 31);
                int phys = idx < 32 ? pa : pb;
                if (has && (phys < 0 || phys >= prm.num_blocks)) {
                    record_error(prm.err, PK_ERR_BAD_INDEX);
                    phys = 0;
                }
                const int y = (phys * Hkv + it.kvh) * bs + (k0 - blk * bs);
                const uint32_t nload = (uint32_t)__popc(__ballot_sync(0xffffffffu, has));
                const int valid_keys = it.c - j * kUKeys;  // warp-uniform
                const bool tail = is_v && valid_keys < kUKeys;
                uint8_t *dst = is_v ? sm + G::OffV + (size_t)s * G::VBytes
                                    : sm + G::OffK + (size_t)s * G::KBytes + p * G::KPanel;
                uint64_t *bar = tail ? v_tma : &full[s];
                if (lane == 0) {
                    if (nload == 0) mbar_arrive(bar);  // keys past the context: nothing to load
                    else mbar_arrive_expect_tx(bar, nload * (is_v ? G::VBlock : 2048u));
                }
                __syncwarp();
                // lane jb issues block jb's box: a warp's TMA instructions issue one
                // at a time, so eight lanes start a stage's boxes together
                if (has) {
                    if (is_v) tma_load_3d(dst + lane * G::VBlock, &tmv3, 0, y, 0, bar);
                    else tma_load_2d(dst + lane * 2048, &tmk2, p * 64, y, bar);
                }
                __syncwarp();
                if (tail) {
                    // V rows past the context (stale or never loaded) must be zero, P
                    // is 0 there: once the stage's V has landed, zero them, then
                    // release the stage to the MMA thread
                    const bool landed = mbar_wait(v_tma, (uint32_t)ntail & 1);
                    ++ntail;
                    if (!landed) {
                        ok = false;
                        break;
                    }
                    for (int i = lane; i < (kUKeys - valid_keys) * (D / 8); i += 32) {
                        const int key = valid_keys + i / (D / 8), ch = i % (D / 8);
                        *(uint4 *)(dst + (key >> 4) * G::VBlock + (ch >> 3) * 2048 + (key & 15) * 128 + (ch & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[s]);
                }
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
        uint8_t *qbuf = sm + G::OffQ + t * G::QBytes;
        int n = 0, n_item = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && idx < n_items;
             idx = snake_next(idx, blockIdx.x, gridDim.x), ++n_item) {
            UItem it;
            item_of(idx, it);
            const int R = it.rt * kUItemRows + t * kURows + r;
            const bool valid = R < it.rows;
            const int tok = valid ? R / g : 0, hh = valid ? R % g : 0;
            const int pos = it.c - it.qn + tok;
            const long long qrow = ((long long)(it.qs0 + tok) * Hq + it.kvh * g + hh) * D;
            // Q row into the K-major 128-byte-swizzled layout (the previous item's
            // MMAs have completed: its o_full was seen)
            {
                const uint4 *src = (const uint4 *)(prm.q + qrow);
#pragma unroll
                for (int ch = 0; ch < D / 8; ++ch) {
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
                if (!mbar_wait(B.s_full, (uint32_t)n & 1)) {
                    ok = false;
                    break;
                }
                tc_after();
                uint32_t sa[64], sb[64];
                tmem_ld64(row_t + s_col, sa);
                tmem_ld64(row_t + s_col + 64u, sb);
                tmem_wait_ld();
                const int k0 = j * kUKeys;
                // scores in log2 units are s * scale_log2; the running max is kept in
                // those units, the raw max (scale > 0) is taken first, in eight
                // interleaved chains (the row sum below uses four partial sums).
                // Stages wholly below every row's diagonal skip the mask.
                if (!__all_sync(0xffffffffu, valid && k0 + kUKeys - 1 <= pos)) {
#pragma unroll
                    for (int i = 0; i < 64; ++i) {
                        if (!(valid && k0 + i <= pos)) sa[i] = __float_as_uint(-INFINITY);
                        if (!(valid && k0 + 64 + i <= pos)) sb[i] = __float_as_uint(-INFINITY);
                    }
                }
                float mt[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mt[i] = fmaxf(__uint_as_float(sa[i]), __uint_as_float(sb[i]));
#pragma unroll
                for (int i = 8; i < 64; ++i)
                    mt[i & 7] = fmax3(mt[i & 7], __uint_as_float(sa[i]), __uint_as_float(sb[i]));
                mt[0] = fmax3(mt[0], mt[1], mt[2]);
                mt[3] = fmax3(mt[3], mt[4], mt[5]);
                mt[0] = fmax3(mt[0], mt[3], fmaxf(mt[6], mt[7]));
                const float mx = mt[0] * prm.scale_log2;
                float alpha = 1.f;
                bool resc = false;
                if (__any_sync(0xffffffffu, mx > m + kURescaleLog2)) {
                    const float mn = fmaxf(m, mx);
                    alpha = mn == -INFINITY ? 1.f : fast_exp2(m - mn);
                    resc = j > 0;  // O holds earlier stages
                    m = mn;
                    l *= alpha;
                }
                const float bm = m == -INFINITY ? 0.f : m;
                const float sl = prm.scale_log2;
                const uint64_t sl2 = f2_pack(sl, sl), nbm2 = f2_pack(-bm, -bm);
                uint64_t ps2[2] = {0ull, 0ull};  // two packed partial sums (0.f, 0.f)
                // P as bf16 over the first 64 columns of S: keys 16c..16c+15 in
                // columns 8c..8c+7, two keys per column, the even one in the low half
#pragma unroll
                for (int c = 0; c < kUBlk; ++c) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int key = 16 * c + 2 * i;
                        const float x0 = __uint_as_float(key < 64 ? sa[key] : sb[key - 64]);
                        const float x1 = __uint_as_float(key + 1 < 64 ? sa[key + 1] : sb[key + 1 - 64]);
                        const uint64_t y = f2_fma(f2_pack(x0, x1), sl2, nbm2);  // x * scale - m, log2 units
                        float y0, y1;
                        f2_unpack(y, y0, y1);
                        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                        ps2[i & 1] = f2_add(ps2[i & 1], f2_pack(p0, p1));
                        pk[i] = pack_bf16(p0, p1);
                    }
                    tmem_st8(row_t + s_col + (uint32_t)(8 * c), pk);
                }
                {
                    float a0, a1, b0, b1;
                    f2_unpack(ps2[0], a0, a1);
                    f2_unpack(ps2[1], b0, b1);
                    l += (a0 + a1) + (b0 + b1);
                }
                if (resc) {  // O_t is stable: its last P V completed before this S did
#pragma unroll 1
                    for (int q8 = 0; q8 < D / 16; ++q8) {
                        uint32_t ov[16];
                        tmem_ld16(row_t + o_col + (uint32_t)(q8 * 16), ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st16(row_t + o_col + (uint32_t)(q8 * 16), ov);
                    }
                }
                tmem_wait_st();
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
            for (int q4 = 0; q4 < D / 32; ++q4) {
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
            // O_t += P_t V of stage nn (first: the item's first stage, which
            // overwrites O_t once the previous item's epilogue has read it)
            auto pv = [&](int t, int nn, bool first) -> bool {
                const UTileBars B = tb(t);
                if (!mbar_wait(B.p_full, (uint32_t)nn & 1)) return false;
                if (first && n_item > 0 && !mbar_wait(B.o_free, (uint32_t)(n_item - 1) & 1)) return false;
                const int s = nn % kUVStages;
                if (t == 0 && !mbar_wait(&v_full[s], (uint32_t)(nn / kUVStages) & 1)) return false;
                tc_after();
                const uint32_t vlo = sdesc_lo(smem_u32(sm + G::OffV + (size_t)s * G::VBytes), 2048);
#pragma unroll
                for (int kp = 0; kp < kUBlk; ++kp)
                    umma_ts(tmem + 256u + (uint32_t)(t * 128), tmem + (uint32_t)(t * 128 + 8 * kp),
                            vlo + kp * (G::VBlock >> 4), G::IdescPV, (first && kp == 0) ? 0u : 1u);
                return true;
            };
            // S_t = Q_t K^T of the stage in K slot s, over S_t's (and P_t's) columns
            auto s_mma = [&](int t, int s) {
                const uint32_t klo = sdesc_lo(smem_u32(sm + G::OffK + (size_t)s * G::KBytes), 16);
                const uint32_t qlo = sdesc_lo(smem_u32(sm + G::OffQ + t * G::QBytes), 16);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)  // 16-column K-steps, four per 64-column panel
                    umma_ss(tmem + (uint32_t)(t * 128), qlo + (uint32_t)((kk >> 2) * (kURows * 128) + (kk & 3) * 32) / 16,
                            klo + (uint32_t)((kk >> 2) * G::KPanel + (kk & 3) * 32) / 16, kIdescS, kk > 0 ? 1u : 0u);
                umma_commit(tb(t).s_full);
            };
            for (int idx = blockIdx.x; ok && idx < n_items;
                 idx = snake_next(idx, blockIdx.x, gridDim.x), ++n_item) {
                UItem it;
                item_of(idx, it);
                for (int t = 0; t < kUTiles && ok; ++t) ok = mbar_wait(tb(t).q_full, (uint32_t)n_item & 1);
                if (!ok) break;
                for (int j = 0; j < it.nkt; ++j, ++n) {
                    const int s = n % kUKStages;
                    if (!mbar_wait(&k_full[s], (uint32_t)(n / kUKStages) & 1) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    for (int t = 0; t < kUTiles; ++t) {
                        // P_t V of the previous stage, then S_t of this one in the same columns
                        if (j > 0 && !pv(t, n - 1, j == 1)) {
                            ok = false;
                            break;
                        }
                        s_mma(t, s);
                    }
                    if (!ok) break;
                    umma_commit(&k_empty[s]);  // the K slot is free once both S have completed
                    if (j > 0) umma_commit(&v_empty[(n - 1) % kUVStages]);
                }
                if (!ok) break;
                for (int t = 0; t < kUTiles && ok; ++t) {
                    ok = pv(t, n - 1, it.nkt == 1);
                    if (ok) umma_commit(tb(t).o_full);
                }
                if (!ok) break;
                umma_commit(&v_empty[(n - 1) % kUVStages]);
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

template <int D>
int umma_prepare(pk_pool *p, bool &ok) {
    ok = false;
    cudaError_t ce = cudaFuncSetAttribute(attention_chunk_umma_kernel<D>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, (int)UGeo<D>::Smem);
    if (ce != cudaSuccess) return cuda_fail(ce, "set chunk (tcgen05) smem size");
    // the warpgroups' register split assumes this launch register count
    cudaFuncAttributes fa;
    ce = cudaFuncGetAttributes(&fa, attention_chunk_umma_kernel<D>);
    if (ce != cudaSuccess) return cuda_fail(ce, "chunk (tcgen05) attributes");
    ok = fa.numRegs == kURegLaunch;
    return PK_OK;
}

}  // namespace

// Serves bf16 pools with 16-row tile boxes (block_size a multiple of 16) and
// groups dividing 128: this kernel at head dim 64 or 128, the head-dim-256
// kernel (attention_chunk_umma256.cu) at 256, where two 128-row tiles would need
// 2 x (128 S + 256 O) tensor-memory columns of the 512.  PK_CHUNK_MMA_SYNC=1
// selects the mma.sync chunk kernel instead.
int chunk_umma_prepare_pool(pk_pool *p) {
    p->umma_ok = p->umma256_ok = false;
    const char *e = getenv("PK_CHUNK_MMA_SYNC");
    if (!p->tile_map3d || (e && e[0] == '1')) return PK_OK;
    if (p->head_dim != 64 && p->head_dim != 128 && p->head_dim != 256) return PK_OK;
    bool ok = false;
    int rc = PK_OK;
    if (p->head_dim == 256) {
        rc = chunk_umma256_prepare(p);
        ok = rc == PK_OK;
    } else {
        rc = p->head_dim == 64 ? umma_prepare<64>(p, ok) : umma_prepare<128>(p, ok);
    }
    if (rc != PK_OK || !ok) return rc;
    // K as 2-D 16-row boxes of one 64-column panel; V uses the pool's 3-D tile map
    const int rc2 = encode_pool_map(&p->tmap_k2, p->k_base, p, kTile);
    if (rc2 != PK_OK) return rc2;
    if (p->head_dim == 256) p->umma256_ok = true;
    else p->umma_ok = true;
    return PK_OK;
}

bool chunk_umma_applies(const pk_pool *p, const AttnArgs &a) {
    const int g = a.n_q_heads / p->n_kv_heads;
    return (p->umma_ok || p->umma256_ok) && g >= 1 && kURows % g == 0;
}

int launch_chunk_umma(const pk_pool *p, const AttnArgs &a, bool all_multi, cudaStream_t st) {
    if (p->head_dim == 256) return launch_chunk_umma256(p, a, all_multi, st);
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
    u.min_rows = all_multi ? u.group : kTile;
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        u.seq0 = s0;
        u.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        const cudaError_t e =
            p->head_dim == 64
                ? launch_dependent(attention_chunk_umma_kernel<64>, dim3(p->sm_count), kUThreads, UGeo<64>::Smem, st,
                                   p->tmap_k2, p->tmap_v, u)
                : launch_dependent(attention_chunk_umma_kernel<128>, dim3(p->sm_count), kUThreads, UGeo<128>::Smem,
                                   st, p->tmap_k2, p->tmap_v, u);
        if (e != cudaSuccess) return cuda_fail(e, "chunk attention (tcgen05) launch");
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "chunk attention (tcgen05) launch");
}

}  // namespace pk
