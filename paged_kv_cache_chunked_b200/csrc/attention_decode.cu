// Paged decode attention on the tensor cores for bf16 pools (head_dim
// 64/128/256, block_size a multiple of 8): every sequence whose query rows
// fit one 16-row MMA tile (q_b * g <= 16: decodes, and chunks of a few
// tokens).  Chunks with more rows run in the chunk kernel.
//
// What is computed ["PagedAttention & Continuous Batching" (study notes),
// "Block tables"; "Batching and PagedAttention", "PagedAttention" item 4]:
// for query token i of sequence b (position p = c_b - q_b + i) and q head h,
// softmax attention over keys 0..p of kv head h / g, key j read from physical
// block table_b[j / bs] at slot j % bs.
//
// Structure.  Each warp is an independent pipeline: it claims work items (one
// row tile of one (sequence, kv head) against one partition of the context)
// from a global counter, stages the item's Q rows by bulk copy, and streams
// the item's 16-token KV tiles with TMA through its own ring of shared-memory
// stages, keeping kStages - 1 tiles in flight while it computes one.  A TMA
// load is issued per warp here because one issuing warp sustains only about
// 14 GB/s of scattered 2-4 KiB tile loads on B200; six issuing warps per SM
// saturate HBM where one producer warp per CTA could not.  S = Q K^T and
// O += P V run on mma.sync m16n8k16 (bf16 in, fp32 accumulate) with an
// online softmax in fp32 registers.  The context of a sequence is cut into
// partitions (flash-decoding-style split-K) so that the batch yields about
// kItemsPerCta items per resident CTA; the warp that finishes the last
// partition of a (sequence, kv head) merges the partitions' (O, log2-sum-exp)
// into the output, found by an arrival counter.
//
// Every wait is bounded (2 s); on expiry the kernel records PK_ERR_TIMEOUT,
// waits (bounded) for its own copies in flight and returns.  Block ids are
// range-checked before use.
#include "tc_common.cuh"

#include <algorithm>

namespace pk {
namespace {

using namespace tc;

constexpr int kItemsPerCta = 12;  // split-K target: items per resident CTA

template <int D>
struct DecCfg;
template <>
struct DecCfg<64> {
    static constexpr int kWarps = 4, kStages = 5, kMinBlocks = 2, kQSlots = 2;
    static constexpr bool kQReg = true;
};
template <>
struct DecCfg<128> {
    static constexpr int kWarps = 3, kStages = 3, kMinBlocks = 2, kQSlots = 2;
    static constexpr bool kQReg = true;
};
template <>
struct DecCfg<256> {
    static constexpr int kWarps = 4, kStages = 2, kMinBlocks = 1, kQSlots = 1;
    static constexpr bool kQReg = false;
};

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// One warp's item, written by the warp's lane 0 next to the item's Q rows.
struct Desc {
    int seq, kvh, kv_begin, kv_end, nparts, row, part_base, pstride, c, qn, qs0, rows;
};

template <int D>
struct DecSmem {
    using C = DecCfg<D>;
    static constexpr int kStageBytes = 64 * D;  // K then V: 16 rows x D x 2 bytes each
    static constexpr size_t kRing = 0;
    static constexpr size_t kQBuf = kRing + (size_t)C::kWarps * C::kStages * kStageBytes;
    static constexpr size_t kQPriv = kQBuf + (size_t)C::kWarps * C::kQSlots * 32 * D;
    static constexpr size_t kPlan = kQPriv + (C::kQReg ? 0 : (size_t)C::kWarps * 32 * D);
    static constexpr size_t kDesc = kPlan + align_up(5 * (size_t)kPlanLen * 4, 16);
    static constexpr size_t kBars = kDesc + align_up(sizeof(Desc) * C::kWarps * C::kQSlots, 16);
    static constexpr size_t kEnd = kBars + (size_t)C::kWarps * (C::kStages + C::kQSlots) * 8;
    static constexpr size_t kBytes = kEnd + 1024;  // + alignment slack
};

template <int D>
constexpr int dec_threads() { return DecCfg<D>::kWarps * 32; }

struct DecParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables;
    const int32_t *ctx, *qsl;
    int seq0, nseq;
    int max_blocks, n_q_heads, n_kv_heads, group, block_size, box_rows, num_blocks, num_tokens;
    int ncta, cap_rows;
    bool map3d;  // tensor maps are 3-D: one box per 16-row tile
    float scale_log2;
    WsHeader *hdr;
    int *counters;                   // per (sequence in the window, kv head)
    float *partial_o, *partial_lse;  // [row][D], [row]
    int *err;
};

// T8: every item is one decode token of a group of at most 8 q heads.  The
// heads then sit on the N = 8 side of the MMA (S^T = K Q^T, O^T = V^T P^T):
// half the MMAs and half the accumulator registers of the 16-row layout,
// with P^T moved into B-fragment order by movmatrix.
template <int D, bool T8>
__global__ void __launch_bounds__(dec_threads<D>(), DecCfg<D>::kMinBlocks)
attention_decode_kernel(const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const DecParams prm) {
    using C = DecCfg<D>;
    using L = DecSmem<D>;
    constexpr int S = C::kStages, QS = C::kQSlots;
    constexpr int KS = D / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hkv = prm.n_kv_heads, g = prm.group, Hq = prm.n_q_heads;
    PlanArrays pa;
    pa.split_pre = (int *)(sm + L::kPlan);
    pa.rows_pre = pa.split_pre + kPlanLen;
    pa.prow_pre = pa.rows_pre + kPlanLen;
    pa.s_qsl = pa.prow_pre + kPlanLen;
    pa.s_ctx = pa.s_qsl + kPlanLen;
    uint64_t *full = (uint64_t *)(sm + L::kBars) + (size_t)warp * (S + QS);
    uint64_t *qfull = full + S;
    uint8_t *ring = sm + L::kRing + (size_t)warp * S * L::kStageBytes;
    uint8_t *qbuf = sm + L::kQBuf + (size_t)warp * QS * 32 * D;
    uint8_t *qpriv = sm + L::kQPriv + (size_t)warp * 32 * D;
    Desc *descs = (Desc *)(sm + L::kDesc) + (size_t)warp * QS;

    __shared__ int s_nsplit;
    if (lane == 0) {
        for (int s = 0; s < S + QS; ++s) mbar_init(&full[s], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        PlanArgs a;
        a.qsl = prm.qsl;
        a.ctx = prm.ctx;
        a.seq0 = prm.seq0;
        a.nseq = prm.nseq;
        a.num_tokens = prm.num_tokens;
        a.block_size = prm.block_size;
        a.max_blocks = prm.max_blocks;
        a.group = g;
        a.n_kv_heads = Hkv;
        a.ncta = prm.ncta;
        a.items_per_cta = kItemsPerCta;
        a.rows_group = 1;
        a.cap_rows = prm.cap_rows;
        a.err = prm.err;
        const PlanTotals t = plan_window(a, pa, lane);
        if (lane == 0) s_nsplit = t.n_split;
    }
    __syncthreads();
    const int n_items = s_nsplit;
    const int nseq = prm.nseq, bs = prm.block_size, box = prm.box_rows;

    // ------------------------------------------------------------ producer side
    // An item is staged (claimed, its Q rows bulk-copied, its descriptor and
    // first table chunk taken) as soon as one of the warp's kQSlots Q slots is
    // free, i.e. a whole item ahead of its use; its KV tiles are issued
    // kStages ahead of the consumer in stream order.  The next claim is always
    // in flight, so the atomic's latency hides too.
    auto claim = [&]() -> int {
        int v = 0;
        if (lane == 0) v = atomicAdd(&prm.hdr->next_item, 1);
        return v;  // lane 0 only; broadcast when used
    };
    auto chunk_entry = [&](int b, int blk_base) -> int {
        const int nblk = (pa.s_ctx[b] + bs - 1) / bs;
        const int e = blk_base + lane;
        return e < nblk ? __ldg(prm.tables + (long long)(prm.seq0 + b) * prm.max_blocks + e) : 0;
    };
    int pending = claim();
    bool ok = true, exhausted = false;
    int n_iss = 0, n_con = 0, n_staged = 0, n_begun = 0, n_started = 0;
    uint32_t qph = 0;        // parity bit per Q slot (consumer side)
    int tab_s0 = 0, tab_s1 = 0;  // each staged item's first table chunk (this lane's entry);
                                 // loaded straight into the slot's register so the load
                                 // stays in flight until the item starts
    // producer cursor
    bool p_active = false;
    int p_b = 0, p_kvh = 0, p_kt = 0, p_ke = 0, p_c = 0;
    int cur_base = 0, cur_tab = 0, nxt_tab = 0;

    auto table_get = [&](int blk) -> int {
        while (blk >= cur_base + 32) {  // move to the prefetched chunk, prefetch the next
            cur_base += 32;
            cur_tab = nxt_tab;
            nxt_tab = chunk_entry(p_b, cur_base + 32);
        }
        int phys = __shfl_sync(0xffffffffu, cur_tab, blk - cur_base);
        if (phys < 0 || phys >= prm.num_blocks) {
            if (lane == 0) record_error(prm.err, PK_ERR_BAD_INDEX);
            phys = 0;
        }
        return phys;
    };
    auto stage_next = [&]() {
        const int idx = __shfl_sync(0xffffffffu, pending, 0);
        if (idx >= n_items) {
            exhausted = true;
            return;
        }
        pending = claim();
        const SplitItem it = decode_split(pa, nseq, g, Hkv, idx);
        const int slot = n_staged % QS;
        const int qs0 = pa.s_qsl[it.b], qn = pa.s_qsl[it.b + 1] - qs0;
        if (slot == 0) tab_s0 = chunk_entry(it.b, (it.kv_begin * kTile / bs) & ~31);
        else tab_s1 = chunk_entry(it.b, (it.kv_begin * kTile / bs) & ~31);
        if (lane == 0) {
            Desc &d = descs[slot];
            d.seq = prm.seq0 + it.b;
            d.kvh = it.kvh;
            d.kv_begin = it.kv_begin;
            d.kv_end = it.kv_end;
            d.nparts = it.nparts;
            d.row = it.part_base + it.part * it.pstride;
            d.part_base = it.part_base;
            d.pstride = it.pstride;
            d.c = pa.s_ctx[it.b];
            d.qn = qn;
            d.qs0 = qs0;
            d.rows = it.rows;
            mbar_arrive_expect_tx(&qfull[slot], (uint32_t)it.rows * D * 2);
        }
        __syncwarp();
        // the item's rows (token-major, heads of the group contiguous per token):
        // one contiguous run of g heads per query token, lane t copies token t
        if (lane < qn)
            bulk_load(qbuf + (size_t)slot * 32 * D + (size_t)lane * g * D * 2,
                      prm.q + ((long long)(qs0 + lane) * Hq + it.kvh * g) * D, (uint32_t)g * D * 2,
                      &qfull[slot]);
        ++n_staged;
    };
    auto start_item = [&]() {
        const int slot = n_started % QS;
        const Desc &d = descs[slot];
        p_b = d.seq - prm.seq0;
        p_kvh = d.kvh;
        p_kt = d.kv_begin;
        p_ke = d.kv_end;
        p_c = d.c;
        cur_base = (p_kt * kTile / bs) & ~31;
        cur_tab = slot == 0 ? tab_s0 : tab_s1;
        nxt_tab = chunk_entry(p_b, cur_base + 32);
        p_active = true;
        ++n_started;
    };
    auto issue_tile = [&]() {
        const int stage = n_iss % S;
        const int kt = p_kt;
        int y0 = 0, y1 = 0, nsub = 0;
        for (int t0 = kt * kTile; t0 < kt * kTile + kTile && t0 < p_c; t0 += box) {
            const int y = (table_get(t0 / bs) * Hkv + p_kvh) * bs + t0 % bs;
            if (nsub == 0) y0 = y; else y1 = y;
            ++nsub;
        }
        if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], (uint32_t)nsub * 2 * (D / 64) * box * 128);
            uint8_t *ks = ring + (size_t)stage * L::kStageBytes;
            uint8_t *vs = ks + 32 * D;
            if (prm.map3d) {  // one box per tile: 16 rows of every panel
                tma_load_3d(ks, &tmk, 0, y0, 0, &full[stage]);
                tma_load_3d(vs, &tmv, 0, y0, 0, &full[stage]);
            }
            for (int sb = 0; sb < (prm.map3d ? 0 : nsub); ++sb) {
                const int y = sb == 0 ? y0 : y1;
#pragma unroll
                for (int pn = 0; pn < D / 64; ++pn) {
                    tma_load_2d(ks + pn * 2048 + sb * box * 128, &tmk, pn * 64, y, &full[stage]);
                    tma_load_2d(vs + pn * 2048 + sb * box * 128, &tmv, pn * 64, y, &full[stage]);
                }
            }
        }
        __syncwarp();
        ++n_iss;
        if (++p_kt == p_ke) p_active = false;
    };
    auto refill = [&]() {
        while (!exhausted && n_staged - n_begun < QS) stage_next();
        while (n_iss - n_con < S) {
            if (!p_active) {
                if (n_started == n_staged) break;
                start_item();
            }
            issue_tile();
        }
    };

    // ------------------------------------------------------------ consumer side
    const int qr = lane >> 2, qc = (lane & 3) * 2;
    const int mi = lane >> 3, rr = lane & 7;
    const int k_row = (mi >> 1) * 8 + rr, k_col = (mi & 1) * 8;  // K (B of Q K^T)
    const int v_row = (mi & 1) * 8 + rr, v_col = (mi >> 1) * 8;  // V (B of P V, transposed)
    const int q_row = (mi & 1) * 8 + rr, q_col = (mi >> 1) * 8;  // Q (A of Q K^T)
    int c_kt = 0, c_ke = 0;  // consumer's position in its current item
    int c = 0, lim0 = 0, lim1 = 0, d_seq = 0, d_kvh = 0, d_nparts = 1, d_row = 0, d_base = 0,
        d_pstride = 0, d_qs0 = 0, d_rows = 0;
    long long orow0 = -1, orow1 = -1;
    uint32_t qf[(C::kQReg && !T8) ? KS : 1][4];
    float o[T8 ? 1 : D / 8][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    // T8 state: Q^T as B fragments, O^T accumulators (16 d-rows x 8 heads per
    // m-tile), running max / sum for heads qc and qc + 1
    uint32_t qb[T8 ? KS : 1][2];
    float ot[T8 ? KS : 1][4];

    auto begin_item = [&]() {
        const int slot = n_begun % QS;
        if (!mbar_wait(&qfull[slot], (qph >> slot) & 1)) {
            ok = false;
            return;
        }
        qph ^= 1u << slot;
        const Desc &d = descs[slot];
        c = d.c;
        c_kt = d.kv_begin;
        c_ke = d.kv_end;
        d_seq = d.seq;
        d_kvh = d.kvh;
        d_nparts = d.nparts;
        d_row = d.row;
        d_base = d.part_base;
        d_pstride = d.pstride;
        d_qs0 = d.qs0;
        d_rows = d.rows;
        const int qn = d.qn, rows = d.rows;
        const int r0 = qr, r1 = qr + 8;
        lim0 = r0 < rows ? c - qn + r0 / g : c - 1;
        lim1 = r1 < rows ? c - qn + r1 / g : c - 1;
        orow0 = r0 < rows ? (long long)(d_qs0 + r0 / g) * Hq + d_kvh * g + r0 % g : -1;
        orow1 = r1 < rows ? (long long)(d_qs0 + r1 / g) * Hq + d_kvh * g + r1 % g : -1;
        const uint8_t *qs = qbuf + (size_t)slot * 32 * D;
        if constexpr (T8) {
            const int h = lane >> 2;  // the B fragment's n index: head of the group
            const uint8_t *qh = qs + h * D * 2;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int col = (kk * 16 + qc) * 2;
                qb[kk][0] = h < rows ? *(const uint32_t *)(qh + col) : 0u;
                qb[kk][1] = h < rows ? *(const uint32_t *)(qh + col + 16) : 0u;
            }
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) ot[mt][0] = ot[mt][1] = ot[mt][2] = ot[mt][3] = 0.f;
        } else if constexpr (C::kQReg) {
            const uint8_t *q0 = qs + qr * D * 2, *q1 = qs + (qr + 8) * D * 2;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int col = (ks * 16 + qc) * 2;
                qf[ks][0] = r0 < rows ? *(const uint32_t *)(q0 + col) : 0u;
                qf[ks][1] = r1 < rows ? *(const uint32_t *)(q1 + col) : 0u;
                qf[ks][2] = r0 < rows ? *(const uint32_t *)(q0 + col + 16) : 0u;
                qf[ks][3] = r1 < rows ? *(const uint32_t *)(q1 + col + 16) : 0u;
            }
        } else {
            for (int ch = lane; ch < 16 * (D / 8); ch += 32) {
                const int row = ch / (D / 8), col = (ch % (D / 8)) * 8;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (row < rows) v = *(const uint4 *)(qs + (row * D + col) * 2);
                *(uint4 *)(qpriv + swz(row, col)) = v;
            }
        }
        __syncwarp();
        ++n_begun;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    };

    auto compute_tile = [&](int kt, uint8_t *ks, uint8_t *vs) {
        const int valid = c - kt * kTile;  // tokens of this tile inside the context
        if (valid < kTile) {
            // tail tile: clear V rows past the context (stale or never-written slots)
            for (int ch = lane; ch < (kTile - valid) * (D / 8); ch += 32) {
                const int row = valid + ch / (D / 8), col = (ch % (D / 8)) * 8;
                *(uint4 *)(vs + swz(row, col)) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async();  // the stage is rewritten by TMA later
            __syncwarp();
        }
        const uint32_t ka = smem_u32(ks), va = smem_u32(vs), qa = smem_u32(qpriv);
        if constexpr (T8) {
            // S^T (16 tokens x 8 heads): A = K rows, B = Q^T
            float st[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(ka + swz(q_row, kk * 16 + q_col), a0, a1, a2, a3);
                mma_bf16(st, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
            }
            // st[0], st[1]: token qr, heads qc, qc + 1; st[2], st[3]: token qr + 8
            const int tok0 = kt * kTile + qr;
            float s0 = st[0] * prm.scale_log2, s1 = st[1] * prm.scale_log2;
            float s2 = st[2] * prm.scale_log2, s3 = st[3] * prm.scale_log2;
            if (tok0 >= c) s0 = s1 = -INFINITY;
            if (tok0 + 8 >= c) s2 = s3 = -INFINITY;
            float ma = fmaxf(s0, s2), mb = fmaxf(s1, s3);
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, x));
                mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, x));
            }
            const float na = fmaxf(m0, ma), nb = fmaxf(m1, mb);
            const float ba = na == -INFINITY ? 0.f : na, bb = nb == -INFINITY ? 0.f : nb;
            const float ala = fast_exp2(m0 - ba), alb = fast_exp2(m1 - bb);
            m0 = na;
            m1 = nb;
            const float p0 = fast_exp2(s0 - ba), p1 = fast_exp2(s1 - bb);
            const float p2 = fast_exp2(s2 - ba), p3 = fast_exp2(s3 - bb);
            l0 = l0 * ala + p0 + p2;
            l1 = l1 * alb + p1 + p3;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                ot[mt][0] *= ala;
                ot[mt][1] *= alb;
                ot[mt][2] *= ala;
                ot[mt][3] *= alb;
            }
            // P^T as the B fragment: transpose the two 8x8 (token x head) blocks
            const uint32_t b0 = movmatrix_trans(pack_bf16(p0, p1));
            const uint32_t b1 = movmatrix_trans(pack_bf16(p2, p3));
            // O^T (16 d-rows x 8 heads per m-tile) += V^T P^T
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4_t(va + swz(k_row, mt * 16 + k_col), a0, a1, a2, a3);
                mma_bf16(ot[mt], a0, a1, a2, a3, b0, b1);
            }
            return;
        }
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            uint32_t a0, a1, a2, a3;
            if constexpr (C::kQReg) {
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

    auto finish_item = [&]() {
        if constexpr (T8) {
            // sums over the 16 token lanes of each head
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                l0 += __shfl_xor_sync(0xffffffffu, l0, x);
                l1 += __shfl_xor_sync(0xffffffffu, l1, x);
            }
            const float ia = l0 > 0.f ? 1.f / l0 : 0.f, ib = l1 > 0.f ? 1.f / l1 : 0.f;
            const int ha = qc, hb = qc + 1;  // heads of this lane's accumulators
            const bool va_ = ha < d_rows, vb_ = hb < d_rows;
            if (d_nparts <= 1) {
                __nv_bfloat16 *oa = prm.out + ((long long)d_qs0 * Hq + d_kvh * g + ha) * D;
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
                return;
            }
            float *pa_ = prm.partial_o + (size_t)(d_row + ha) * D;
            float *pb_ = pa_ + D;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const int d0 = mt * 16 + qr;
                if (va_) {
                    pa_[d0] = ot[mt][0] * ia;
                    pa_[d0 + 8] = ot[mt][2] * ia;
                }
                if (vb_) {
                    pb_[d0] = ot[mt][1] * ib;
                    pb_[d0 + 8] = ot[mt][3] * ib;
                }
            }
            if (qr == 0) {
                float *pl = prm.partial_lse + (size_t)d_row;
                if (va_) pl[ha] = l0 > 0.f ? m0 + __log2f(l0) : -INFINITY;
                if (vb_) pl[hb] = l1 > 0.f ? m1 + __log2f(l1) : -INFINITY;
            }
        } else {
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
        }  // 16-row layout
        __threadfence();
        __syncwarp();
        int prev = 0;
        int *cnt = prm.counters + (size_t)(d_seq - prm.seq0) * Hkv + d_kvh;
        if (lane == 0) prev = atomicAdd(cnt, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        if (prev != d_nparts - 1) return;
        // last partition of (sequence, kv head): merge all partitions into the output
        __threadfence();
        merge_partials<D>(prm.partial_o, prm.partial_lse, d_base, d_pstride, d_nparts, 0,
                          min(kTile, d_rows), prm.out, d_qs0, Hq, d_kvh, g, lane);
        if (lane == 0) *cnt = 0;  // leave the counter zeroed for the next call
    };

    // ------------------------------------------------------------ main loop
    refill();
    while (ok && n_con < n_iss) {
        if (c_kt >= c_ke) {
            begin_item();
            if (!ok) break;
            refill();  // stage the item after next now that a Q slot is free
        }
        const int stage = n_con % S;
        if (!mbar_wait(&full[stage], (uint32_t)(n_con / S) & 1)) {
            ok = false;
            break;
        }
        uint8_t *ks = ring + (size_t)stage * L::kStageBytes;
        compute_tile(c_kt, ks, ks + 32 * D);
        ++n_con;
        if (++c_kt == c_ke) finish_item();
        refill();
    }
    if (!ok) {
        if (lane == 0) record_error(prm.err, PK_ERR_TIMEOUT);
        // never leave with a copy still writing into this CTA's shared memory
        for (int n = n_con; n < n_iss; ++n) mbar_wait(&full[n % S], (uint32_t)(n / S) & 1);
        for (int k = n_begun; k < n_staged; ++k) mbar_wait(&qfull[k % QS], (qph >> (k % QS)) & 1);
    }
    __syncthreads();
    release_counter(prm.hdr);
}

}  // namespace

// ------------------------------------------------------------------ host side
int dec_threads_of(int D) {
    switch (D) {
        case 64: return dec_threads<64>();
        case 128: return dec_threads<128>();
        default: return dec_threads<256>();
    }
}

template <int D, bool T8>
static int dec_prepare_one(int *per_sm) {
    const int smem = (int)DecSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(attention_decode_kernel<D, T8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "set decode attention smem size");
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, attention_decode_kernel<D, T8>,
                                                      dec_threads<D>(), smem);
    if (e != cudaSuccess) return cuda_fail(e, "decode attention occupancy");
    return PK_OK;
}

template <int D>
static int dec_prepare(pk_pool *p) {
    int a = 0, b = 0;
    int rc = dec_prepare_one<D, false>(&a);
    if (rc == PK_OK) rc = dec_prepare_one<D, true>(&b);
    if (rc != PK_OK) return rc;
    const int per_sm = std::min(a, b);
    if (per_sm < 1) return fail(PK_ERR_UNSUPPORTED, "decode attention kernel does not fit on an SM");
    p->tc_ctas = per_sm * p->sm_count;
    return PK_OK;
}

int decode_prepare_pool(pk_pool *p) {
    switch (p->head_dim) {
        case 64: return dec_prepare<64>(p);
        case 128: return dec_prepare<128>(p);
        case 256: return dec_prepare<256>(p);
        default: return fail(PK_ERR_UNSUPPORTED, "decode path: head_dim %d", p->head_dim);
    }
}

int decode_items_per_cta() { return kItemsPerCta; }

template <int D>
static int dec_launch(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, cudaStream_t st) {
    DecParams tp;
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
    tp.map3d = p->tile_map3d;
    tp.num_blocks = p->num_blocks;
    tp.num_tokens = a.num_tokens;
    tp.ncta = p->tc_ctas;
    tp.cap_rows = w.cap_rows;
    tp.scale_log2 = a.scale * 1.4426950408889634f;
    tp.hdr = (WsHeader *)w.header;
    tp.counters = w.counters;
    tp.partial_o = w.partial_o;
    tp.partial_lse = w.partial_lse;
    tp.err = p->d_err;
    // every query token its sequence's only one and a group of <= 8 heads: the
    // decode-specialised layout; anything else (short chunks, larger groups) the
    // 16-row layout
    const bool t8 = a.num_tokens == a.num_seqs && tp.group <= 8;
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        tp.seq0 = s0;
        tp.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        if (t8)
            attention_decode_kernel<D, true><<<p->tc_ctas, dec_threads<D>(), DecSmem<D>::kBytes, st>>>(
                p->tmap_k, p->tmap_v, tp);
        else
            attention_decode_kernel<D, false><<<p->tc_ctas, dec_threads<D>(), DecSmem<D>::kBytes, st>>>(
                p->tmap_k, p->tmap_v, tp);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "decode attention launch");
}

int launch_decode(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, cudaStream_t st) {
    switch (p->head_dim) {
        case 64: return dec_launch<64>(p, a, w, st);
        case 128: return dec_launch<128>(p, a, w, st);
        case 256: return dec_launch<256>(p, a, w, st);
        default: return fail(PK_ERR_UNSUPPORTED, "decode path: head_dim %d", p->head_dim);
    }
}

}  // namespace pk
