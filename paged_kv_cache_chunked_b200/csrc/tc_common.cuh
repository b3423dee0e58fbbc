// Device helpers shared by the two tensor-core attention kernels (decode and
// chunk): PTX wrappers, the shared-memory swizzle, and the work planner.
#pragma once

#include <cuda_bf16.h>

#include "pk_internal.h"

namespace pk {
namespace tc {

constexpr unsigned long long kWaitNs = 2000000000ull;  // bounded wait: 2 s
constexpr int kPlanLen = kMaxSeqsPerLaunch + 1;
constexpr int kPartitionMinTiles = 4;  // smallest split-K partition (64 tokens)

// Workspace header of one kernel (must start zeroed; every call leaves it zeroed).
struct WsHeader {
    int next_item;  // dynamic scheduler: next item to claim
    int done;       // CTAs finished (the last one resets both fields)
    int pad[62];
};

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
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}
// The same with an L2 cache policy (l2_evict_first_policy for data read once).
__device__ __forceinline__ void tma_load_3d_hint(void *dst, const CUtensorMap *map, int x, int y, int z,
                                                 uint64_t *bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)), "l"(pol)
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
// An L2 policy for data read once (the K/V stream of a decode launch): its
// lines are the first to be evicted, so the stream does not push out the
// launch's reused lines (block tables, queries, split-K partial rows).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// An L2 policy under which the lines a store writes are the last to be
// evicted: rows written early in a launch and read back at its end (split-K
// partial rows) then survive the stream of K/V reads in between.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void st_l2_keep(float *dst, float v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(dst), "f"(v), "l"(pol) : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}
// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA / bulk copy) writes to the same memory.
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
// Transpose of an 8x8 matrix of 16-bit elements held in MMA fragment order
// (lane l holds row l / 4, columns 2 (l % 4) and 2 (l % 4) + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
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

// Smallest i in [0, n) with pre[i + 1] > idx (pre: inclusive scan, pre[0] = 0).
__device__ __forceinline__ int find_seq(const int *pre, int n, int idx) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid + 1] > idx) hi = mid; else lo = mid + 1;
    }
    return lo;
}

// ---------------------------------------------------------------- planning
// Work of one window of sequences, derived identically by every CTA.
//   split sequences (q_b * g <= 16, i.e. decodes): the context's 16-token KV
//     tiles are cut into ceil(tiles / P) partitions, one item per (partition,
//     kv head); P is chosen so that the window yields about items_per_cta
//     items per resident CTA, and coarsened until the split-K partial rows fit
//     the workspace;
//   rows sequences (chunks): ceil(row tiles / rows_group) items per kv head.
// Arrays (inclusive prefix sums over the window's sequences, [0] = 0):
//   split_pre (split items), rows_pre (rows items), prow_pre (partial rows),
//   s_qsl (query start lens, window-relative index), s_ctx (context lens).
struct PlanArgs {
    const int32_t *qsl, *ctx;
    int seq0, nseq, num_tokens, block_size, max_blocks, group, n_kv_heads;
    int ncta, items_per_cta, rows_group, cap_rows;
    int *err;
};

struct PlanArrays {
    int *split_pre, *rows_pre, *prow_pre, *s_qsl, *s_ctx;
};

struct PlanTotals {
    int n_split, n_rows;
};

// Executed by one full warp.
__device__ inline PlanTotals plan_window(const PlanArgs &a, const PlanArrays &p, int lane) {
    const int nseq = a.nseq, g = a.group, Hkv = a.n_kv_heads;
    auto valid = [&](int s0, int s1, int c) {
        const int qn = s1 - s0;
        return s0 >= 0 && s1 <= a.num_tokens && qn >= 1 && c >= qn &&
               (long long)(c + a.block_size - 1) / a.block_size <= a.max_blocks;
    };
    unsigned long long tiles = 0;
    for (int i = lane; i < nseq; i += 32) {
        const int b = a.seq0 + i;
        const int s0 = __ldg(a.qsl + b), s1 = __ldg(a.qsl + b + 1), c = __ldg(a.ctx + b);
        p.s_qsl[i] = s0;
        p.s_ctx[i] = c;
        if (i == nseq - 1) p.s_qsl[nseq] = s1;
        if (!valid(s0, s1, c)) record_error(a.err, PK_ERR_BAD_INDEX);
        else if ((s1 - s0) * g <= kTile) tiles += (c + kTile - 1) / kTile;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, o);
    __syncwarp();  // s_qsl / s_ctx written by other lanes are read below
    const unsigned long long want = (unsigned long long)a.ncta * a.items_per_cta;
    unsigned long long P = (tiles * Hkv + want - 1) / want;
    if (P < kPartitionMinTiles) P = kPartitionMinTiles;
    PlanTotals t{0, 0};
    for (int attempt = 0; attempt < 8; ++attempt) {
        int run_s = 0, run_r = 0, run_p = 0;
        for (int base = 0; base < nseq; base += 32) {
            const int i = base + lane;
            int ns = 0, nr = 0, np = 0;
            if (i < nseq) {
                const int c = p.s_ctx[i], qn = p.s_qsl[i + 1] - p.s_qsl[i];
                if (valid(p.s_qsl[i], p.s_qsl[i + 1], c)) {
                    if (qn * g <= kTile) {
                        const int kt = (c + kTile - 1) / kTile;
                        const int nparts = (int)(((unsigned long long)kt + P - 1) / P);
                        ns = nparts * Hkv;
                        np = nparts > 1 ? nparts * Hkv * qn * g : 0;
                    } else {
                        const int rtiles = (qn * g + kTile - 1) / kTile;
                        nr = (rtiles + a.rows_group - 1) / a.rows_group * Hkv;
                    }
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
                p.split_pre[i + 1] = run_s + is;
                p.rows_pre[i + 1] = run_r + ir;
                p.prow_pre[i + 1] = run_p + ip;
            }
            run_s += __shfl_sync(0xffffffffu, is, 31);
            run_r += __shfl_sync(0xffffffffu, ir, 31);
            run_p += __shfl_sync(0xffffffffu, ip, 31);
        }
        t.n_split = run_s;
        t.n_rows = run_r;
        if (run_p <= a.cap_rows) break;
        // more split-K partial rows than the workspace holds (chunks of a few
        // tokens): coarser partitions, finally one partition per sequence
        P = attempt < 6 ? 2 * P : (1ull << 40);
    }
    if (lane == 0) {
        p.split_pre[0] = 0;
        p.rows_pre[0] = 0;
        p.prow_pre[0] = 0;
    }
    __syncwarp();
    return t;
}

// A split item decoded from its index (window-relative sequence b).
struct SplitItem {
    int b, kvh, part, nparts, kv_begin, kv_end, rows, part_base, pstride;
};

__device__ inline SplitItem decode_split(const PlanArrays &p, int nseq, int group, int Hkv, int j) {
    SplitItem it;
    const int b = find_seq(p.split_pre, nseq, j);
    const int local = j - p.split_pre[b];
    it.b = b;
    it.kvh = local % Hkv;
    it.part = local / Hkv;
    it.nparts = (p.split_pre[b + 1] - p.split_pre[b]) / Hkv;
    const int kt = (p.s_ctx[b] + kTile - 1) / kTile;
    it.kv_begin = (int)((long long)it.part * kt / it.nparts);
    it.kv_end = (int)((long long)(it.part + 1) * kt / it.nparts);
    it.rows = (p.s_qsl[b + 1] - p.s_qsl[b]) * group;
    // partial rows of partition p: part_base + p * pstride .. + rows - 1
    it.pstride = Hkv * it.rows;
    it.part_base = p.prow_pre[b] + it.kvh * it.rows;
    return it;
}

// Merges the split-K partitions of one (sequence, kv head) into the output
// [flash-decoding combination of per-partition softmax results]:
//   out_r = sum_p 2^(lse_p,r - M_r) o_p,r / sum_p 2^(lse_p,r - M_r),  M_r = max_p lse_p,r
// where o_p,r is partition p's normalised output row r and lse_p,r its
// log2-sum-exp (-inf for a partition with no key).  Partition p's rows sit at
// partial rows base + p * pstride + r; row r is query token r / g (of the
// tokens starting at qs0), q head kvh * g + r % g.  Merges rows row0 ..
// row0 + nrows - 1.  Rows go four at a time, and
// loads are issued for all four rows (and two partitions) at once so their
// latencies overlap.  Executed by one full warp.
template <int D, int UNROLL = 2>
__device__ inline void merge_partials(const float *partial_o, const float *partial_lse, int base,
                                      int pstride, int nparts, int row0, int nrows,
                                      __nv_bfloat16 *out, int qs0, int Hq, int kvh, int g,
                                      int lane) {
    constexpr int RG = 4;
    base += row0;
    for (int r0 = 0; r0 < nrows; r0 += RG) {
        float Mr[RG], den[RG];
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float mx = -INFINITY;
            if (r0 + r < nrows)
                for (int p = lane; p < nparts; p += 32)
                    mx = fmaxf(mx, __ldcg(partial_lse + (size_t)(base + p * pstride) + r0 + r));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            Mr[r] = mx;
        }
#pragma unroll
        for (int r = 0; r < RG; ++r) {
            float sm = 0.f;
            if (r0 + r < nrows)
                for (int p = lane; p < nparts; p += 32) {
                    const float lse = __ldcg(partial_lse + (size_t)(base + p * pstride) + r0 + r);
                    sm += lse == -INFINITY ? 0.f : fast_exp2(lse - Mr[r]);
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
            den[r] = sm > 0.f ? 1.f / sm : 0.f;
        }
        for (int c4 = lane; c4 < D / 4; c4 += 32) {
            float4 acc[RG];
#pragma unroll
            for (int r = 0; r < RG; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll UNROLL
            for (int p = 0; p < nparts; ++p) {
                const size_t prow = (size_t)(base + p * pstride) + r0;
#pragma unroll
                for (int r = 0; r < RG; ++r) {
                    if (r0 + r < nrows) {
                        const float lse = __ldcg(partial_lse + prow + r);
                        const float wgt = lse == -INFINITY ? 0.f : fast_exp2(lse - Mr[r]);
                        const float4 x = __ldcg((const float4 *)(partial_o + (prow + r) * D) + c4);
                        acc[r].x += wgt * x.x;
                        acc[r].y += wgt * x.y;
                        acc[r].z += wgt * x.z;
                        acc[r].w += wgt * x.w;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RG; ++r) {
                if (r0 + r < nrows) {
                    const int row = row0 + r0 + r;
                    const long long orow = (long long)(qs0 + row / g) * Hq + kvh * g + row % g;
                    uint2 pk;
                    pk.x = pack_bf16(acc[r].x * den[r], acc[r].y * den[r]);
                    pk.y = pack_bf16(acc[r].z * den[r], acc[r].w * den[r]);
                    *(uint2 *)(out + orow * D + c4 * 4) = pk;
                }
            }
        }
    }
}

// The last CTA to finish resets the work counter for the next call (call
// after a __syncthreads that every thread of the CTA reaches).
__device__ inline void release_counter(WsHeader *hdr) {
    if (threadIdx.x == 0) {
        __threadfence();
        const int d = atomicAdd(&hdr->done, 1);
        if (d == (int)gridDim.x - 1) {
            hdr->next_item = 0;
            hdr->done = 0;
            __threadfence();
        }
    }
}

}  // namespace tc
}  // namespace pk
