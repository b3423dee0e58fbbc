// Paged attention for causal prefill chunks on the tensor cores (bf16 pools,
// head_dim 64/128/256, block_size a multiple of 8): every sequence whose
// query rows (q_b tokens x g heads of a kv group) span more than one 16-row
// MMA tile.  Decodes and chunks of a few tokens run in the decode kernel.
//
// What is computed ["Batching and PagedAttention", "Continuous batching":
// long prompts are split into chunks across steps; "PagedAttention & Continuous
// Batching" (study notes), "Block tables"]: query token i of a chunk of q
// tokens at context c sits at position c - q + i and attends to keys 0..c-q+i
// of its kv head, each key read through the sequence's block table.
//
// Structure.  A work item is NC x RT row tiles (16 rows each: pairs (query
// token, head of the group), token-major) of one (sequence, kv head).  One
// producer warp per CTA claims items from a global counter, stages each
// consumer warp's Q rows by bulk copy, and streams every visible 16-token KV
// tile of the item by TMA through a ring of shared-memory stages; all NC
// consumer warps compute on every stage, each for its own RT row tiles (the KV
// tile is loaded once per NC x RT row tiles, and each warp loads its K and V
// fragments once for its RT tiles), masking causally by its own rows.
// S = Q K^T and O += P V run on mma.sync m16n8k16 with an online softmax in
// fp32 registers.  Bounded waits as in the decode kernel.
#include "tc_common.cuh"

#include <algorithm>

namespace pk {
namespace {

using namespace tc;

constexpr int kTagAll = 15;  // stage consumed by every consumer warp
constexpr int kTagEnd = -1;  // no more stages
constexpr int kFirst = 1, kLast = 2;

constexpr float kRescaleLog2 = 8.f;  // lazy softmax rescale threshold (log2 units)

template <int D>
struct ChunkCfg;
// One CTA per SM with 7 consumer warps of RT row tiles each: every KV tile
// the producer warp loads feeds 7 x RT row tiles (224 query rows at RT = 2).
// The producer's TMA issue rate, not the tensor pipe, bounds this kernel, so
// the rows a tile feeds set its speed.  Eight warps keep 255 registers per
// thread available; at RT = 2 the Q fragments come from shared memory.
template <>
struct ChunkCfg<64> {
    static constexpr int kStages = 16, kMinBlocks = 1, kConsumers = 7, kRowTiles = 2;
    static constexpr bool kQReg = false;
};
template <>
struct ChunkCfg<128> {
    static constexpr int kStages = 12, kMinBlocks = 1, kConsumers = 7, kRowTiles = 2;
    static constexpr bool kQReg = false;
};
template <>
struct ChunkCfg<256> {
    static constexpr int kStages = 8, kMinBlocks = 1, kConsumers = 4, kRowTiles = 1;
    static constexpr bool kQReg = false;
};

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct RowDesc {
    int seq, kvh, tile, kv_end, c, qn, qs0, rows;
};

template <int D>
struct ChunkSmem {
    using C = ChunkCfg<D>;
    static constexpr int kStageBytes = 64 * D;
    static constexpr size_t kRing = 0;
    static constexpr size_t kQStage = kRing + (size_t)C::kStages * kStageBytes;
    static constexpr size_t kQPriv = kQStage + (size_t)C::kConsumers * C::kRowTiles * 32 * D;
    static constexpr size_t kPlan =
        kQPriv + (C::kQReg ? 0 : (size_t)C::kConsumers * C::kRowTiles * 32 * D);
    static constexpr size_t kDesc = kPlan + align_up(5 * (size_t)kPlanLen * 4, 16);
    static constexpr size_t kBars = kDesc + align_up(C::kConsumers * sizeof(RowDesc), 16);
    static constexpr size_t kMeta = kBars + (size_t)(2 * C::kStages + 2 * C::kConsumers) * 8;
    static constexpr size_t kFlag = kMeta + (size_t)C::kStages * 16;
    static constexpr size_t kEnd = kFlag + 16;
    static constexpr size_t kBytes = kEnd + 1024;
};

template <int D>
constexpr int chunk_threads() { return (ChunkCfg<D>::kConsumers + 1) * 32; }

struct ChunkParams {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    const int32_t *tables;
    const int32_t *ctx, *qsl;
    int seq0, nseq;
    int max_blocks, n_q_heads, n_kv_heads, group, block_size, box_rows, num_blocks, num_tokens;
    bool map3d;  // tensor maps are 3-D: one box per 16-row tile
    float scale_log2;
    WsHeader *hdr;
    int *err;
};

template <int D>
__global__ void __launch_bounds__(chunk_threads<D>(), ChunkCfg<D>::kMinBlocks)
attention_chunk_kernel(const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const ChunkParams prm) {
    using C = ChunkCfg<D>;
    using L = ChunkSmem<D>;
    constexpr int S = C::kStages, NC = C::kConsumers, RT = C::kRowTiles;
    constexpr int KS = D / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint64_t *full = (uint64_t *)(sm + L::kBars);
    uint64_t *empty = full + S;
    uint64_t *qfull = empty + S;
    uint64_t *qempty = qfull + NC;
    int4 *meta = (int4 *)(sm + L::kMeta);
    volatile int *abort_flag = (volatile int *)(sm + L::kFlag);
    RowDesc *descs = (RowDesc *)(sm + L::kDesc);
    PlanArrays pa;
    pa.split_pre = (int *)(sm + L::kPlan);
    pa.rows_pre = pa.split_pre + kPlanLen;
    pa.prow_pre = pa.rows_pre + kPlanLen;
    pa.s_qsl = pa.prow_pre + kPlanLen;
    pa.s_ctx = pa.s_qsl + kPlanLen;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hkv = prm.n_kv_heads, g = prm.group, Hq = prm.n_q_heads;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NC);
        }
        for (int w = 0; w < NC; ++w) {
            mbar_init(&qfull[w], 1);
            mbar_init(&qempty[w], 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == NC) {
        // ================================================================ producer warp
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
        a.ncta = 1;
        a.items_per_cta = 1;
        a.rows_group = NC * RT;
        a.cap_rows = 1 << 30;  // split items are not this kernel's work
        a.err = nullptr;       // the decode kernel reports bad sequences
        const PlanTotals t = plan_window(a, pa, lane);
        const int n_rows = t.n_rows, nseq = prm.nseq, bs = prm.block_size, box = prm.box_rows;

        int stage = 0;
        uint32_t phase = 0, qphase = 0;
        uint32_t armed = 0, armed_parity = 0;  // per stage: ever armed, parity of last phase
        bool ok = true;
        int pending = 0;
        if (lane == 0) pending = atomicAdd(&prm.hdr->next_item, 1);
        for (;;) {
            const int idx = __shfl_sync(0xffffffffu, pending, 0);
            if (idx >= n_rows || !ok) break;
            if (lane == 0) pending = atomicAdd(&prm.hdr->next_item, 1);
            const int b = find_seq(pa.rows_pre, nseq, idx);
            const int local = idx - pa.rows_pre[b];
            const int kvh = local % Hkv, grp = local / Hkv;
            const int c = pa.s_ctx[b], qs0 = pa.s_qsl[b], qn = pa.s_qsl[b + 1] - qs0;
            const int rows_total = qn * g;
            const int last_row = min((grp + 1) * NC * RT * kTile, rows_total) - 1;
            const int kv_end = (c - qn + last_row / g) / kTile + 1;
            // Q rows and descriptor of each consumer warp's row tile
            for (int w = 0; w < NC && ok; ++w) {
                if (!mbar_wait(&qempty[w], ((qphase >> w) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                qphase ^= 1u << w;
                const int tile = (grp * NC + w) * RT, r0 = tile * kTile;  // the warp's first row tile
                const int nrows = max(0, min(RT * kTile, rows_total - r0));
                if (lane == 0) {
                    RowDesc &d = descs[w];
                    d.seq = prm.seq0 + b;
                    d.kvh = kvh;
                    d.tile = nrows > 0 ? tile : -1;
                    d.kv_end = kv_end;
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
                        bulk_load(sm + L::kQStage + (size_t)w * RT * 32 * D + (size_t)(ra - r0) * D * 2,
                                  prm.q + ((long long)(qs0 + t) * Hq + kvh * g + (ra - t * g)) * D,
                                  (uint32_t)(rb - ra) * D * 2, &qfull[w]);
                    }
                }
                __syncwarp();
            }
            // every visible KV tile, for all consumer warps
            const int32_t *table = prm.tables + (long long)(prm.seq0 + b) * prm.max_blocks;
            const int nblk = (c + bs - 1) / bs;
            int base = 0;
            int cur = lane < nblk ? __ldg(table + lane) : 0;
            int nxt = 32 + lane < nblk ? __ldg(table + 32 + lane) : 0;
            for (int kt = 0; kt < kv_end && ok; ++kt) {
                if (!mbar_wait(&empty[stage], phase ^ 1)) {
                    ok = false;
                    break;
                }
                int y0 = 0, y1 = 0, nsub = 0;
                for (int t0 = kt * kTile; t0 < kt * kTile + kTile && t0 < c; t0 += box) {
                    const int blk = t0 / bs;
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
                    const int y = (phys * Hkv + kvh) * bs + t0 % bs;
                    if (nsub == 0) y0 = y; else y1 = y;
                    ++nsub;
                }
                if (lane == 0) {
                    meta[stage] = make_int4(kTagAll, kt, (kt == 0 ? kFirst : 0) | (kt == kv_end - 1 ? kLast : 0), 0);
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)nsub * 2 * (D / 64) * box * 128);
                    uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
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
                armed |= 1u << stage;
                armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // end marker
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
        const int qr = lane >> 2, qc = (lane & 3) * 2;
        const int mi = lane >> 3, rr = lane & 7;
        const int k_row = (mi >> 1) * 8 + rr, k_col = (mi & 1) * 8;
        const int v_row = (mi & 1) * 8 + rr, v_col = (mi >> 1) * 8;
        const int q_row = (mi & 1) * 8 + rr, q_col = (mi >> 1) * 8;
        const uint8_t *qstage = sm + L::kQStage + (size_t)w * RT * 32 * D;
        uint8_t *qpriv = sm + L::kQPriv + (size_t)w * RT * 32 * D;  // RT swizzled 16-row tiles

        int stage = 0;
        uint32_t phase = 0, qph = 0;
        bool active = false, ok = true;
        int c = 0, max_lim = 0;
        // per row tile t: rows qr and qr + 8 (limits, output rows, softmax state)
        int lim0[RT], lim1[RT];
        long long orow0[RT], orow1[RT];
        uint32_t qf[C::kQReg ? KS : 1][4];
        float o[RT][D / 8][4];
        float m0[RT], m1[RT], l0[RT], l1[RT];

        auto begin_item = [&]() {
            if (!mbar_wait(&qfull[w], qph)) {
                ok = false;
                return;
            }
            qph ^= 1;
            const RowDesc &d = descs[w];
            active = d.tile >= 0;
            c = d.c;
            const int rows = d.rows, qn = d.qn;
            const int tile0 = max(d.tile, 0);
            max_lim = c - qn + (min((tile0 + RT) * kTile, rows) - 1) / g;
#pragma unroll
            for (int t = 0; t < RT; ++t) {
                const int tile = tile0 + t;
                const int r0 = tile * kTile + qr, r1 = r0 + 8;
                // rows past the last query row compute garbage that is never written
                lim0[t] = r0 < rows ? c - qn + r0 / g : c - 1;
                lim1[t] = r1 < rows ? c - qn + r1 / g : c - 1;
                orow0[t] = active && r0 < rows ? (long long)(d.qs0 + r0 / g) * Hq + d.kvh * g + r0 % g : -1;
                orow1[t] = active && r1 < rows ? (long long)(d.qs0 + r1 / g) * Hq + d.kvh * g + r1 % g : -1;
                const int nvalid = active ? max(0, min(kTile, rows - tile * kTile)) : 0;
                const uint8_t *qs = qstage + (size_t)t * 32 * D;
                if constexpr (C::kQReg) {
                    const uint8_t *q0 = qs + qr * D * 2, *q1 = qs + (qr + 8) * D * 2;
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const int col = (ks * 16 + qc) * 2;
                        qf[ks][0] = qr < nvalid ? *(const uint32_t *)(q0 + col) : 0u;
                        qf[ks][1] = qr + 8 < nvalid ? *(const uint32_t *)(q1 + col) : 0u;
                        qf[ks][2] = qr < nvalid ? *(const uint32_t *)(q0 + col + 16) : 0u;
                        qf[ks][3] = qr + 8 < nvalid ? *(const uint32_t *)(q1 + col + 16) : 0u;
                    }
                } else {
                    uint8_t *qp = qpriv + (size_t)t * 32 * D;
                    for (int ch = lane; ch < 16 * (D / 8); ch += 32) {
                        const int row = ch / (D / 8), col = (ch % (D / 8)) * 8;
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (row < nvalid) v = *(const uint4 *)(qs + (row * D + col) * 2);
                        *(uint4 *)(qp + swz(row, col)) = v;
                    }
                }
#pragma unroll
                for (int n = 0; n < D / 8; ++n) o[t][n][0] = o[t][n][1] = o[t][n][2] = o[t][n][3] = 0.f;
                m0[t] = m1[t] = -INFINITY;
                l0[t] = l1[t] = 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[w]);
        };

        auto finish_item = [&]() {
            if (!active) return;
#pragma unroll
            for (int t = 0; t < RT; ++t) {
                float a0 = l0[t], a1 = l1[t];
                a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
                a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
                a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
                a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
                const float inv0 = a0 > 0.f ? 1.f / a0 : 0.f, inv1 = a1 > 0.f ? 1.f / a1 : 0.f;
                if (orow0[t] >= 0) {
                    __nv_bfloat16 *dst = prm.out + orow0[t] * D;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n)
                        *(uint32_t *)(dst + n * 8 + qc) = pack_bf16(o[t][n][0] * inv0, o[t][n][1] * inv0);
                }
                if (orow1[t] >= 0) {
                    __nv_bfloat16 *dst = prm.out + orow1[t] * D;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n)
                        *(uint32_t *)(dst + n * 8 + qc) = pack_bf16(o[t][n][2] * inv1, o[t][n][3] * inv1);
                }
            }
        };

        auto compute_tile = [&](int kt, uint8_t *ks, uint8_t *vs) {
            const int valid = c - kt * kTile;
            if (valid < kTile) {
                // tail tile: clear V rows past the context (every warp writes the same zeros)
                for (int ch = lane; ch < (kTile - valid) * (D / 8); ch += 32) {
                    const int row = valid + ch / (D / 8), col = (ch % (D / 8)) * 8;
                    *(uint4 *)(vs + swz(row, col)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
                __syncwarp();
            }
            const uint32_t ka = smem_u32(ks), va = smem_u32(vs), qa = smem_u32(qpriv);
            // S = Q K^T per row tile; each K fragment serves all RT tiles; two
            // accumulator chains per 8-key half (even / odd k-steps)
            float sc[RT][2][4], sd[RT][2][4];
#pragma unroll
            for (int t = 0; t < RT; ++t)
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int i = 0; i < 4; ++i) sc[t][h][i] = sd[t][h][i] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(ka + swz(k_row, kk * 16 + k_col), b0, b1, b2, b3);
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    uint32_t a0, a1, a2, a3;
                    if constexpr (C::kQReg) {
                        a0 = qf[kk][0];
                        a1 = qf[kk][1];
                        a2 = qf[kk][2];
                        a3 = qf[kk][3];
                    } else {
                        ldsm_x4(qa + t * 32 * D + swz(q_row, kk * 16 + q_col), a0, a1, a2, a3);
                    }
                    if (kk & 1) {
                        mma_bf16(sd[t][0], a0, a1, a2, a3, b0, b1);
                        mma_bf16(sd[t][1], a0, a1, a2, a3, b2, b3);
                    } else {
                        mma_bf16(sc[t][0], a0, a1, a2, a3, b0, b1);
                        mma_bf16(sc[t][1], a0, a1, a2, a3, b2, b3);
                    }
                }
            }
            const int key0 = kt * kTile + qc;
            uint32_t pf[RT][4];  // P as A fragments, per row tile
#pragma unroll
            for (int t = 0; t < RT; ++t) {
                const bool full_tile = kt * kTile + kTile - 1 <= min(lim0[t], lim1[t]);
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float sv = (sc[t][nt][i] + sd[t][nt][i]) * prm.scale_log2;
                        if (!full_tile) {
                            const int key = key0 + nt * 8 + (i & 1);
                            if (key > (i < 2 ? lim0[t] : lim1[t])) sv = -INFINITY;
                        }
                        sc[t][nt][i] = sv;
                        if (i < 2) mx0 = fmaxf(mx0, sv); else mx1 = fmaxf(mx1, sv);
                    }
                // Lazy rescaling: the row reference m moves (and O, l are rescaled)
                // only when a score exceeds it by more than kRescaleLog2, so
                // 2^(s - m) stays below 2^kRescaleLog2; o = O / l is exact for any
                // reference.  The vote keeps the branch warp-uniform.
                if (__any_sync(0xffffffffu, mx0 > m0[t] + kRescaleLog2 || mx1 > m1[t] + kRescaleLog2)) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                    const float mn0 = fmaxf(m0[t], mx0), mn1 = fmaxf(m1[t], mx1);
                    const float al0 = mn0 == -INFINITY ? 1.f : fast_exp2(m0[t] - mn0);
                    const float al1 = mn1 == -INFINITY ? 1.f : fast_exp2(m1[t] - mn1);
                    m0[t] = mn0;
                    m1[t] = mn1;
                    l0[t] *= al0;
                    l1[t] *= al1;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        o[t][n][0] *= al0;
                        o[t][n][1] *= al0;
                        o[t][n][2] *= al1;
                        o[t][n][3] *= al1;
                    }
                }
                const float bb0 = m0[t] == -INFINITY ? 0.f : m0[t], bb1 = m1[t] == -INFINITY ? 0.f : m1[t];
                float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    sc[t][nt][0] = fast_exp2(sc[t][nt][0] - bb0);
                    sc[t][nt][1] = fast_exp2(sc[t][nt][1] - bb0);
                    sc[t][nt][2] = fast_exp2(sc[t][nt][2] - bb1);
                    sc[t][nt][3] = fast_exp2(sc[t][nt][3] - bb1);
                    ps0 += sc[t][nt][0] + sc[t][nt][1];
                    ps1 += sc[t][nt][2] + sc[t][nt][3];
                }
                l0[t] += ps0;
                l1[t] += ps1;
                pf[t][0] = pack_bf16(sc[t][0][0], sc[t][0][1]);
                pf[t][1] = pack_bf16(sc[t][0][2], sc[t][0][3]);
                pf[t][2] = pack_bf16(sc[t][1][0], sc[t][1][1]);
                pf[t][3] = pack_bf16(sc[t][1][2], sc[t][1][3]);
            }
            // O += P V; each V fragment serves all RT tiles
#pragma unroll
            for (int np = 0; np < KS; ++np) {
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(va + swz(v_row, np * 16 + v_col), v0, v1, v2, v3);
#pragma unroll
                for (int t = 0; t < RT; ++t) {
                    mma_bf16(o[t][2 * np], pf[t][0], pf[t][1], pf[t][2], pf[t][3], v0, v1);
                    mma_bf16(o[t][2 * np + 1], pf[t][0], pf[t][1], pf[t][2], pf[t][3], v2, v3);
                }
            }
        };

        for (;;) {
            if (!mbar_wait(&full[stage], phase)) {
                ok = false;
                break;
            }
            const int4 mt = meta[stage];
            if (mt.x == kTagEnd) break;
            if (mt.z & kFirst) begin_item();
            if (!ok) break;
            if (active && mt.y * kTile <= max_lim) {
                uint8_t *ks = sm + L::kRing + (size_t)stage * L::kStageBytes;
                compute_tile(mt.y, ks, ks + 32 * D);
            }
            if (mt.z & kLast) finish_item();
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
    __syncthreads();
    release_counter(prm.hdr);
}

template <int D>
int chunk_prepare_t(pk_pool *p) {
    const int smem = (int)ChunkSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(attention_chunk_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "set chunk attention smem size");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attention_chunk_kernel<D>,
                                                      chunk_threads<D>(), smem);
    if (e != cudaSuccess) return cuda_fail(e, "chunk attention occupancy");
    if (per_sm < 1) return fail(PK_ERR_UNSUPPORTED, "chunk attention kernel does not fit on an SM");
    p->tc_ctas_chunk = per_sm * p->sm_count;
    return PK_OK;
}

template <int D>
int chunk_launch_t(const pk_pool *p, const AttnArgs &a, void *header, cudaStream_t st) {
    ChunkParams tp;
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
    tp.scale_log2 = a.scale * 1.4426950408889634f;
    tp.hdr = (WsHeader *)header;
    tp.err = p->d_err;
    for (int s0 = 0; s0 < a.num_seqs; s0 += kMaxSeqsPerLaunch) {
        tp.seq0 = s0;
        tp.nseq = std::min(kMaxSeqsPerLaunch, a.num_seqs - s0);
        attention_chunk_kernel<D><<<p->tc_ctas_chunk, chunk_threads<D>(), ChunkSmem<D>::kBytes, st>>>(
            p->tmap_k, p->tmap_v, tp);
    }
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "chunk attention launch");
}

}  // namespace

int chunk_prepare_pool(pk_pool *p) {
    switch (p->head_dim) {
        case 64: return chunk_prepare_t<64>(p);
        case 128: return chunk_prepare_t<128>(p);
        case 256: return chunk_prepare_t<256>(p);
        default: return fail(PK_ERR_UNSUPPORTED, "chunk path: head_dim %d", p->head_dim);
    }
}

int launch_chunk(const pk_pool *p, const AttnArgs &a, void *header, cudaStream_t st) {
    switch (p->head_dim) {
        case 64: return chunk_launch_t<64>(p, a, header, st);
        case 128: return chunk_launch_t<128>(p, a, header, st);
        case 256: return chunk_launch_t<256>(p, a, header, st);
        default: return fail(PK_ERR_UNSUPPORTED, "chunk path: head_dim %d", p->head_dim);
    }
}

}  // namespace pk
