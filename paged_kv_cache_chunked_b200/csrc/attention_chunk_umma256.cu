// Paged attention for causal prefill chunks at head dim 256 on the
// fifth-generation tensor cores (tcgen05): bf16 pools, block_size a multiple of
// 16, groups g dividing 128.  It serves the same sequences as the head-dim-128
// chunk kernel (attention_chunk_umma.cu) does at its head dims.
//
// What is computed ["Batching and PagedAttention", "Continuous batching":
// long prompts are split into chunks across steps; "PagedAttention & Continuous
// Batching" (study notes), "Block tables"]: query token i of a chunk of q
// tokens at context c sits at position c - q + i and attends to keys 0..c-q+i
// of its kv head, each key read through the sequence's block table.
//
// Why a kernel of its own.  Tensor memory has 512 columns.  At head dim 256 an
// fp32 O of 128 rows takes 256 of them, so two row tiles (the head-dim-128
// kernel's way of keeping the tensor core busy while a softmax works) do not
// fit.  Here an item is one 128-row tile and the overlap comes from two S
// buffers instead: S of the next 64-key stage is computed while the softmax
// works on this one.  Tensor memory: S buffer b at column 64 b (P over its first
// 32 columns), O at columns 256..511.
//
// Structure.  A work item is 128 query rows (pairs (token, head of the group),
// token-major) of one (sequence, kv head); the CTAs take the items sequence by
// sequence, heaviest sequence first, in the snake order of umma_common.cuh.
// Per 64-key stage:
//   - warp 5 loads K by TMA, one 2-D box per 16-key block and 64-column panel
//     (16 boxes, one per lane) into [panel][64 keys][128 B]; warp 6 loads V, one
//     3-D box per block into [block][panel][16 keys][128 B].  K and V have
//     two-slot rings; a K slot is refilled once its S has completed, a V slot
//     once its P V has.  On a stage that runs past the context the V warp
//     zeroes the rows past it before it releases the stage;
//   - one thread of warp 4 issues, in this order, S_0, S_1, P_0 V, S_2, P_1 V,
//     S_3, ...: S_j = Q K_j^T into buffer j % 2 (M 128, N 64, 16 K-steps) and
//     O += P_j V_j (A = P_j read from tensor memory, B = V MN-major; M 128,
//     N 256, 4 K-steps).  The tensor core runs one thread's MMAs in order, so
//     S_{j+2} overwrites P_j only after P_j V has read it, and when S_j has
//     completed, P_{j-2} V has too;
//   - warps 0..3 own one query row per thread: they read the row of S_j from
//     tensor memory, mask causally, keep the running max m and sum l in fp32
//     (the reference m moves, and O is rescaled in tensor memory, only when a
//     score exceeds it by more than 2^8), and write P_j as packed bf16 over S_j.
//     A rescale of O first waits for P_{j-1} V to complete (a barrier committed
//     after every P V); P_j V waits for the softmax.
// Every wait is bounded (2 s); on expiry the kernel records PK_ERR_TIMEOUT,
// each warp waits (bounded) for its own copies and tensor-core work, and the
// CTA releases its tensor memory and returns.  Block ids are range-checked.
#include "umma_common.cuh"

#include <algorithm>

namespace pk {
namespace {

constexpr int kWD = 256;               // head dim
constexpr int kWRows = 128;            // query rows per item (UMMA M)
constexpr int kWKeys = 64;             // keys per stage (UMMA N of S)
constexpr int kWBlk = kWKeys / 16;     // 16-key blocks per stage
constexpr int kWPanels = kWD / 64;     // 64-column panels: the K producer has a lane per (block, panel)
static_assert(kWBlk * kWPanels <= 32, "one K box per producer lane");
constexpr int kWMma = 4;               // warp 4: tensor memory and MMA issue
constexpr int kWProdK = 5, kWProdV = 6;
constexpr int kWThreads = 7 * 32;      // warps 0..3: softmax and epilogue
constexpr uint32_t kWTmemCols = 512;   // S buffers at 0 and 64, O at 256
constexpr uint32_t kWOCol = 256;
constexpr float kWRescaleLog2 = 8.f;

constexpr uint32_t kWQBytes = kWRows * kWD * 2;      // [panel][128 rows][128 B]
constexpr uint32_t kWKPanel = kWKeys * 128;          // one K panel: 64 keys x 128 B
constexpr uint32_t kWKBytes = kWKeys * kWD * 2;      // [panel][64 keys][128 B]
constexpr uint32_t kWVBlock = 16 * kWD * 2;          // one 16-key block of V: [panel][16 keys][128 B]
constexpr uint32_t kWVBytes = kWKeys * kWD * 2;      // [block][panel][16 keys][128 B]
constexpr uint32_t kWOffQ = 0;
constexpr uint32_t kWOffK = kWOffQ + kWQBytes;
constexpr uint32_t kWOffV = kWOffK + 2 * kWKBytes;
constexpr uint32_t kWOffPlan = kWOffV + 2 * kWVBytes;
constexpr uint32_t kWOffBar = kWOffPlan + ((3 * kPlanLen + kOrderInts) * 4 + 15) / 16 * 16;
// barriers: k_full[2], k_empty[2], v_full[2], v_empty[2], v_tma, s_full[2],
// p_full[2], pv_done, q_full, o_full, o_free, mma_done
constexpr uint32_t kWNumBars = 2 + 2 + 2 + 2 + 1 + 2 + 2 + 1 + 1 + 1 + 1 + 1;
constexpr uint32_t kWOffMisc = kWOffBar + kWNumBars * 8;  // tensor memory address, abort flag
constexpr uint32_t kWSmem = kWOffMisc + 16 + 1024;        // + alignment slack
static_assert(kWSmem <= 227 * 1024 - 64, "chunk kernel (head dim 256) shared memory");

// S = Q K^T: fp32 accumulate, bf16 A and B, K-major both, M = 128, N = 64
constexpr uint32_t kWIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
// O += P V: fp32 accumulate, bf16 A and B, B MN-major, M = 128, N = 256
constexpr uint32_t kWIdescPV =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

struct WParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables, *ctx, *qsl;
    int seq0, nseq, max_blocks, n_q_heads, n_kv_heads, group, block_size, num_blocks, num_tokens;
    int min_rows;  // a sequence is served when its query rows (tokens x group heads) exceed this
    float scale_log2;
    int *err;
};

struct WItem {
    int b, kvh, rt, c, qn, qs0, rows, nkt;
};

__global__ void __launch_bounds__(kWThreads, 1)
attention_chunk_umma256_kernel(const __grid_constant__ CUtensorMap tmk2,  // K: 2-D, 16-row boxes
                               const __grid_constant__ CUtensorMap tmv3,  // V: 3-D, 16 rows x 4 panels
                               const WParams prm) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = prm.group, Hq = prm.n_q_heads, Hkv = prm.n_kv_heads, bs = prm.block_size;
    const int nseq = prm.nseq;
    int *grp_pre = (int *)(sm + kWOffPlan);  // groups (128-row blocks) of sequences 0..i-1
    int *s_qsl = grp_pre + kPlanLen;
    int *s_ctx = s_qsl + kPlanLen;
    const ChunkOrder order(s_ctx + kPlanLen);
    uint64_t *k_full = (uint64_t *)(sm + kWOffBar);
    uint64_t *k_empty = k_full + 2;
    uint64_t *v_full = k_empty + 2;
    uint64_t *v_empty = v_full + 2;
    uint64_t *v_tma = v_empty + 2;
    uint64_t *s_full = v_tma + 1;
    uint64_t *p_full = s_full + 2;
    uint64_t *pv_done = p_full + 2;
    uint64_t *q_full = pv_done + 1;
    uint64_t *o_full = q_full + 1;
    uint64_t *o_free = o_full + 1;
    uint64_t *mma_done = o_free + 1;
    uint32_t *tmem_slot = (uint32_t *)(sm + kWOffMisc);
    volatile int *abort_flag = (volatile int *)(sm + kWOffMisc + 4);
    __shared__ int s_ngroups, s_nchunk;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_full[s], 4);
        }
        mbar_init(v_tma, 1);
        mbar_init(pv_done, 1);
        mbar_init(q_full, 4);
        mbar_init(o_full, 1);
        mbar_init(o_free, 4);
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(kWTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (warp == kWProdK) {
        // groups: every served sequence contributes ceil(rows / 128) groups, each
        // of Hkv items (one per kv head)
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
                if (ok && qn * g > prm.min_rows) n = (qn * g + kWRows - 1) / kWRows;
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
        rank_chunk_seqs<kWRows, kWKeys>(order, s_nchunk, grp_pre, s_qsl, s_ctx, g, Hkv, threadIdx.x, kWThreads);
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

    // the item at position idx of the ranked list (the chunk-sequence count is
    // read back from shared memory: kept in a register across the item loops it
    // would cost the softmax warps a register)
    auto item_of = [&](int idx, WItem &it) {
        int local;
        ranked_item(order, s_nchunk, grp_pre, nseq, Hkv, idx, it.b, local);
        const int nit = grp_pre[it.b + 1] - grp_pre[it.b];
        it.kvh = local / nit;
        it.rt = local - it.kvh * nit;
        it.qs0 = s_qsl[it.b];
        it.qn = s_qsl[it.b + 1] - it.qs0;
        it.c = s_ctx[it.b];
        it.rows = it.qn * g;
        it.nkt = block_stages<kWRows, kWKeys>(it.c, it.qn, g, it.rt);
    };

    if (warp == kWProdK || warp == kWProdV) {
        // ------------------------------------------------------------ producers
        const bool is_v = warp == kWProdV;
        uint64_t *full = is_v ? v_full : k_full;
        uint64_t *empty = is_v ? v_empty : k_empty;
        if (lane == 0) prefetch_tmap(is_v ? &tmv3 : &tmk2);
        int n = 0, ntail = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && idx < n_items;
             idx = snake_next(idx, blockIdx.x, gridDim.x)) {
            WItem it;
            item_of(idx, it);
            const int32_t *table = prm.tables + (long long)(prm.seq0 + it.b) * prm.max_blocks;
            const int nblk = (it.c + bs - 1) / bs;
            int base = 0;
            int cur = lane < nblk ? __ldg(table + lane) : 0;
            int nxt = 32 + lane < nblk ? __ldg(table + 32 + lane) : 0;
            for (int j = 0; j < it.nkt; ++j, ++n) {
                const int s = n & 1;
                if (n >= 2 && !mbar_wait(&empty[s], (uint32_t)((n >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (*abort_flag) {
                    ok = false;
                    break;
                }
                // K: lane l issues block l / 4, panel l % 4 (lanes 0..15); V: lane l
                // issues block l (lanes 0..3).  The table window advances once a
                // stage, to the stage's first block; a stage spans at most 4 blocks,
                // so all of them lie in cur (base..) or nxt (base + 32..)
                const int blk0 = j * kWKeys / bs;  // warp-uniform
                while (blk0 >= base + 32) {
                    base += 32;
                    cur = nxt;
                    nxt = base + 32 + lane < nblk ? __ldg(table + base + 32 + lane) : 0;
                }
                const int jb = is_v ? lane : lane / kWPanels;  // 16-key block of the stage
                const int panel = lane % kWPanels;
                const int k0 = j * kWKeys + jb * 16;
                const bool has = (is_v ? lane < kWBlk : lane < kWPanels * kWBlk) && k0 < it.c;
                const int blk = has ? k0 / bs : blk0;
                const int bidx = blk - base;  // 0 .. 35
                const int pa = __shfl_sync(0xffffffffu, cur, bidx & 31);
                const int pb = __shfl_sync(0xffffffffu, nxt, bidx & 31);
                int phys = bidx < 32 ? pa : pb;
                if (has && (phys < 0 || phys >= prm.num_blocks)) {
                    record_error(prm.err, PK_ERR_BAD_INDEX);
                    phys = 0;
                }
                const int y = (phys * Hkv + it.kvh) * bs + (k0 - blk * bs);
                const uint32_t nbox = (uint32_t)__popc(__ballot_sync(0xffffffffu, has));
                const int valid_keys = it.c - j * kWKeys;  // warp-uniform
                const bool tail = is_v && valid_keys < kWKeys;
                uint8_t *dst = is_v ? sm + kWOffV + (size_t)s * kWVBytes : sm + kWOffK + (size_t)s * kWKBytes;
                uint64_t *bar = tail ? v_tma : &full[s];
                if (lane == 0) {
                    if (nbox == 0) mbar_arrive(bar);  // keys past the context: nothing to load
                    else mbar_arrive_expect_tx(bar, nbox * (is_v ? kWVBlock : 2048u));
                }
                __syncwarp();
                if (has) {
                    if (is_v) tma_load_3d(dst + jb * kWVBlock, &tmv3, 0, y, 0, bar);
                    else tma_load_2d(dst + panel * kWKPanel + jb * 2048, &tmk2, panel * 64, y, bar);
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
                    for (int i = lane; i < (kWKeys - valid_keys) * (kWD / 8); i += 32) {
                        const int key = valid_keys + i / (kWD / 8), ch = i % (kWD / 8);
                        *(uint4 *)(dst + (key >> 4) * kWVBlock + (ch >> 3) * 2048 + (key & 15) * 128 + (ch & 7) * 16) =
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
        for (int m = max(0, n - 2); m < n; ++m) mbar_wait(&full[m & 1], (uint32_t)(m >> 1) & 1);
    } else if (warp < kWMma) {
        // ------------------------------------------------------------ softmax + epilogue
        const int r = warp * 32 + lane;  // the query row this thread owns
        const uint32_t row_t = tmem + ((uint32_t)(warp * 32) << 16);
        uint8_t *qbuf = sm + kWOffQ;
        int n = 0, n_item = 0;
        bool ok = true;
        for (int idx = blockIdx.x; ok && idx < n_items;
             idx = snake_next(idx, blockIdx.x, gridDim.x), ++n_item) {
            WItem it;
            item_of(idx, it);
            const int R = it.rt * kWRows + r;
            const bool valid = R < it.rows;
            const int tok = valid ? R / g : 0, hh = valid ? R % g : 0;
            const int pos = it.c - it.qn + tok;
            const long long qrow = ((long long)(it.qs0 + tok) * Hq + it.kvh * g + hh) * kWD;
            // Q row into the K-major 128-byte-swizzled layout (the previous item's
            // MMAs have completed: its o_full was seen)
            {
                const uint4 *src = (const uint4 *)(prm.q + qrow);
#pragma unroll
                for (int ch = 0; ch < kWD / 8; ++ch) {
                    const uint4 v = valid ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
                    const int pn = ch >> 3, c8 = ch & 7;
                    *(uint4 *)(qbuf + pn * (kWRows * 128) + r * 128 + ((c8 ^ (r & 7)) << 4)) = v;
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(q_full);
            float m = -INFINITY, l = 0.f;
            for (int j = 0; j < it.nkt; ++j, ++n) {
                const int sb = n & 1;
                if (!mbar_wait(&s_full[sb], (uint32_t)(n >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_after();
                uint32_t sa[64];
                tmem_ld64(row_t + (uint32_t)(64 * sb), sa);
                tmem_wait_ld();
                const int k0 = j * kWKeys;
                // stages wholly below every row's diagonal skip the mask
                if (!__all_sync(0xffffffffu, valid && k0 + kWKeys - 1 <= pos)) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (!(valid && k0 + i <= pos)) sa[i] = __float_as_uint(-INFINITY);
                }
                float mt[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mt[i] = fmaxf(__uint_as_float(sa[i]), __uint_as_float(sa[i + 8]));
#pragma unroll
                for (int i = 16; i < 64; i += 16)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mt[k] = fmax3(mt[k], __uint_as_float(sa[i + k]), __uint_as_float(sa[i + 8 + k]));
                mt[0] = fmax3(mt[0], mt[1], mt[2]);
                mt[3] = fmax3(mt[3], mt[4], mt[5]);
                mt[0] = fmax3(mt[0], mt[3], fmaxf(mt[6], mt[7]));
                const float mx = mt[0] * prm.scale_log2;
                float alpha = 1.f;
                bool resc = false;
                if (__any_sync(0xffffffffu, mx > m + kWRescaleLog2)) {
                    const float mn = fmaxf(m, mx);
                    alpha = mn == -INFINITY ? 1.f : fast_exp2(m - mn);
                    resc = j > 0;  // O holds earlier stages
                    m = mn;
                    l *= alpha;
                }
                const float bm = m == -INFINITY ? 0.f : m;
                const float sl = prm.scale_log2;
                const uint64_t sl2 = f2_pack(sl, sl), nbm2 = f2_pack(-bm, -bm);
                uint64_t ps2[2] = {0ull, 0ull};
                // P as bf16 over the first 32 columns of S: keys 16c..16c+15 in
                // columns 8c..8c+7, two keys per column, the even one in the low half
#pragma unroll
                for (int c = 0; c < kWBlk; ++c) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int key = 16 * c + 2 * i;
                        const uint64_t y = f2_fma(f2_pack(__uint_as_float(sa[key]), __uint_as_float(sa[key + 1])),
                                                  sl2, nbm2);
                        float y0, y1;
                        f2_unpack(y, y0, y1);
                        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
                        ps2[i & 1] = f2_add(ps2[i & 1], f2_pack(p0, p1));
                        pk[i] = pack_bf16(p0, p1);
                    }
                    tmem_st8(row_t + (uint32_t)(64 * sb + 8 * c), pk);
                }
                {
                    float a0, a1, b0, b1;
                    f2_unpack(ps2[0], a0, a1);
                    f2_unpack(ps2[1], b0, b1);
                    l += (a0 + a1) + (b0 + b1);
                }
                if (__any_sync(0xffffffffu, resc)) {
                    // O must hold P_{j-1} V before it is rescaled; that MMA was issued
                    // after this row's previous P and before this stage's P V
                    if (!mbar_wait(pv_done, (uint32_t)(n - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    if (resc) {
#pragma unroll 1
                        for (int q16 = 0; q16 < kWD / 16; ++q16) {
                            uint32_t ov[16];
                            tmem_ld16(row_t + kWOCol + (uint32_t)(q16 * 16), ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                            tmem_st16(row_t + kWOCol + (uint32_t)(q16 * 16), ov);
                        }
                    }
                }
                tmem_wait_st();
                tc_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
            }
            if (!ok) break;
            // epilogue: O / l for this thread's row
            if (!mbar_wait(o_full, (uint32_t)n_item & 1)) {
                ok = false;
                break;
            }
            tc_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *dst = (uint4 *)(prm.out + qrow);
#pragma unroll 1
            for (int q32 = 0; q32 < kWD / 32; ++q32) {
                uint32_t ov[32];
                tmem_ld32(row_t + kWOCol + (uint32_t)(q32 * 32), ov);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(ov[8 * c8 + 0]) * inv, __uint_as_float(ov[8 * c8 + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(ov[8 * c8 + 2]) * inv, __uint_as_float(ov[8 * c8 + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(ov[8 * c8 + 4]) * inv, __uint_as_float(ov[8 * c8 + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(ov[8 * c8 + 6]) * inv, __uint_as_float(ov[8 * c8 + 7]) * inv);
                        dst[q32 * 4 + c8] = w;
                    }
                }
            }
            tc_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(o_free);
        }
        if (!ok) {
            if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
            *abort_flag = 1;
        }
    } else if (warp == kWMma) {
        // ------------------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
            bool ok = true;
            int n = 0, n_item = 0;
            const uint32_t qlo = sdesc_lo(smem_u32(sm + kWOffQ), 16);
            // S_m = Q K_m^T into buffer m % 2
            auto s_mma = [&](int mg) -> bool {
                const int s = mg & 1;
                if (!mbar_wait(&k_full[s], (uint32_t)(mg >> 1) & 1) || *abort_flag) return false;
                tc_after();
                const uint32_t klo = sdesc_lo(smem_u32(sm + kWOffK + (size_t)s * kWKBytes), 16);
#pragma unroll
                for (int kk = 0; kk < kWD / 16; ++kk)  // four 16-column K-steps per 64-column panel
                    umma_ss(tmem + (uint32_t)(64 * s), qlo + (uint32_t)((kk >> 2) * (kWRows * 128) + (kk & 3) * 32) / 16,
                            klo + (uint32_t)((kk >> 2) * kWKPanel + (kk & 3) * 32) / 16, kWIdescS, kk > 0 ? 1u : 0u);
                umma_commit(&s_full[s]);
                umma_commit(&k_empty[s]);  // the K slot is free once this S has completed
                return true;
            };
            for (int idx = blockIdx.x; ok && idx < n_items;
                 idx = snake_next(idx, blockIdx.x, gridDim.x), ++n_item) {
                WItem it;
                item_of(idx, it);
                if (!mbar_wait(q_full, (uint32_t)n_item & 1)) {
                    ok = false;
                    break;
                }
                ok = s_mma(n);
                if (ok && it.nkt > 1) ok = s_mma(n + 1);
                for (int j = 0; ok && j < it.nkt; ++j) {
                    const int mg = n + j, s = mg & 1;
                    // O += P_j V_j (first: the item's first stage, which overwrites O
                    // once the previous item's epilogue has read it)
                    if (!mbar_wait(&p_full[s], (uint32_t)(mg >> 1) & 1) ||
                        (j == 0 && n_item > 0 && !mbar_wait(o_free, (uint32_t)(n_item - 1) & 1)) ||
                        !mbar_wait(&v_full[s], (uint32_t)(mg >> 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_after();
                    const uint32_t vlo = sdesc_lo(smem_u32(sm + kWOffV + (size_t)s * kWVBytes), 2048);
#pragma unroll
                    for (int kp = 0; kp < kWBlk; ++kp)
                        umma_ts(tmem + kWOCol, tmem + (uint32_t)(64 * s + 8 * kp), vlo + kp * (kWVBlock >> 4),
                                kWIdescPV, (j == 0 && kp == 0) ? 0u : 1u);
                    umma_commit(&v_empty[s]);
                    umma_commit(pv_done);
                    if (j + 2 < it.nkt) ok = s_mma(mg + 2);
                }
                if (!ok) break;
                umma_commit(o_full);
                n += it.nkt;
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
    if (warp == kWMma) {
        tc_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kWTmemCols)
                     : "memory");
    }
}

}  // namespace

int chunk_umma256_prepare(pk_pool *p) {
    const cudaError_t ce = cudaFuncSetAttribute(attention_chunk_umma256_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWSmem);
    return ce == cudaSuccess ? PK_OK : cuda_fail(ce, "set chunk (tcgen05, head dim 256) smem size");
}

int launch_chunk_umma256(const pk_pool *p, const AttnArgs &a, bool all_multi, cudaStream_t st) {
    WParams u;
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
        const cudaError_t e = launch_dependent(attention_chunk_umma256_kernel, dim3(p->sm_count), kWThreads, kWSmem, st,
                                               p->tmap_k2, p->tmap_v, u);
        if (e != cudaSuccess) return cuda_fail(e, "chunk attention (tcgen05, head dim 256) launch");
    }
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "chunk attention (tcgen05, head dim 256) launch");
}

}  // namespace pk
