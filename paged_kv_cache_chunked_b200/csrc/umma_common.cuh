// tcgen05 helpers shared by the chunk attention kernels: shared-memory matrix
// descriptors, MMA issue with operands in shared or tensor memory, commits to
// mbarriers, tensor-memory loads and stores, and the packed f32x2 arithmetic
// of their softmax warps.  Forms and bit layouts follow the PTX ISA's
// tcgen05 chapter.
#pragma once

#include "tc_common.cuh"

namespace pk {
namespace {

using namespace tc;

// Shared-memory matrix descriptor (128-byte swizzle) as two 32-bit words: the low
// word holds the start address and the leading byte offset (both >> 4), the high
// word the stride byte offset (>> 4, 1024 B here), the descriptor version of
// sm_100 (bit 46 of the 64-bit value) and the swizzle mode (bits 61..63).  The
// MMA thread builds the low word of each operand's base once and adds the
// per-K-step offset (>> 4; addresses stay below 256 KiB, so the 14-bit field
// never carries).
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
constexpr uint32_t kSdescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
// D (tensor memory) [+]= A (shared) x B (shared)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 ad, bd;\n\t"
        "mov.b64 ad, {%1, %5};\n\tmov.b64 bd, {%2, %5};\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, {%6, %6, %6, %6}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kSdescHi), "r"(0u));
}
// D (tensor memory) [+]= A (tensor memory: row m in lane m, two bf16 per column,
// the even K index in the low half) x B (shared)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
        "mov.b64 bd, {%2, %5};\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %3, {%6, %6, %6, %6}, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "r"(kSdescHi), "r"(0u));
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
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :
                 : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
// ---- packed f32x2 arithmetic ----------------------------------------------
// The softmax warps are bound by instruction issue, so their per-key work uses
// the packed two-float forms: one instruction scales and offsets two scores,
// one adds two probabilities to the row sum.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max(a, b, c) in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// ---- order of the work items --------------------------------------------
// A window's chunk work is grouped by sequence; a sequence's items (kv head x
// row block) are taken in their natural order, so that the row blocks of one
// (sequence, kv head), which read the same keys, run side by side and share
// them in L2.  Sequences differ a lot (a chunk at context 4,096 has four times
// the work of one at 1,024), so taking items round robin in sequence order
// leaves the CTAs with the longest sequence's items far behind.  Every CTA
// instead ranks the window's chunk sequences by work, heaviest first (ties by
// index: the same order in every CTA), and CTA i takes the positions of the
// ranked item list in snake order, i, 2P - 1 - i, 2P + i, ... (P CTAs):
// greedy balancing of the longest-first kind, without a shared counter.
// Windows of more than kRankCap chunk sequences, where round robin already
// spreads the work, keep the natural order.
constexpr int kRankCap = 256;
constexpr int kOrderInts = 5 * kRankCap + 1;  // shared-memory ints of a ChunkOrder

struct ChunkOrder {
    int *cseq;       // [kRankCap] chunk sequences (window index), in window order
    int *key;        // [kRankCap] their key stages summed over row blocks
    int *ord;        // [kRankCap] rank -> position in cseq
    int *rank_seq;   // [kRankCap] rank -> window index
    int *rank_pre;   // [kRankCap + 1] items of the ranks before
    __device__ explicit ChunkOrder(int *base)
        : cseq(base), key(base + kRankCap), ord(base + 2 * kRankCap), rank_seq(base + 3 * kRankCap),
          rank_pre(base + 4 * kRankCap) {}
};

// Key stages of row block rt of a chunk of qn tokens at context c: those of its
// last query row (token-major rows of g heads, ROWS rows a block, KEYS keys a
// stage).
template <int ROWS, int KEYS>
__device__ __forceinline__ int block_stages(int c, int qn, int g, int rt) {
    const int last_row = min((rt + 1) * ROWS, qn * g) - 1;
    return (c - qn + last_row / g) / KEYS + 1;
}

// Ranks the m chunk sequences listed in order.cseq (m <= kRankCap) and fills
// order.rank_seq / rank_pre.  grp_pre[i] = row blocks of window sequences
// before i.  Called by every thread of the CTA (it holds barriers).
template <int ROWS, int KEYS>
__device__ void rank_chunk_seqs(const ChunkOrder &o, int m, const int *grp_pre, const int *s_qsl,
                                const int *s_ctx, int g, int Hkv, int tid, int nthreads) {
    for (int j = tid; j < m; j += nthreads) {
        const int b = o.cseq[j];
        const int qn = s_qsl[b + 1] - s_qsl[b], nb = grp_pre[b + 1] - grp_pre[b];
        int w = 0;
        for (int rt = 0; rt < nb; ++rt) w += block_stages<ROWS, KEYS>(s_ctx[b], qn, g, rt);
        o.key[j] = w;
    }
    __syncthreads();
    for (int i = tid; i < m; i += nthreads) {
        const int ki = o.key[i];
        int r = 0;
        for (int j = 0; j < m; ++j) {
            const int kj = o.key[j];
            r += (kj > ki) | ((kj == ki) & (j < i));
        }
        o.ord[r] = i;
    }
    __syncthreads();
    if (tid < 32) {
        int run = 0;
        for (int base = 0; base < m; base += 32) {
            const int r = base + tid;
            int n = 0;
            if (r < m) {
                const int b = o.cseq[o.ord[r]];
                o.rank_seq[r] = b;
                n = (grp_pre[b + 1] - grp_pre[b]) * Hkv;
            }
            int inc = n;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, inc, d);
                if (tid >= d) inc += y;
            }
            if (r < m) o.rank_pre[r + 1] = run + inc;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (tid == 0) o.rank_pre[0] = 0;
    }
}

// The item at position idx of the ranked list (or of the natural list when the
// window has more than kRankCap chunk sequences): window sequence b and its
// local item (kv head x row blocks + row block).
__device__ __forceinline__ void ranked_item(const ChunkOrder &o, int m, const int *grp_pre, int nseq,
                                            int Hkv, int idx, int &b, int &local) {
    if (m <= kRankCap) {
        const int r = find_seq(o.rank_pre, m, idx);
        b = o.rank_seq[r];
        local = idx - o.rank_pre[r];
    } else {
        b = find_seq(grp_pre, nseq, idx / Hkv);
        local = idx - grp_pre[b] * Hkv;
    }
}

// position of CTA cta's item of round r in the ranked list (in
// [r * ncta, (r + 1) * ncta), so strictly increasing in r)
__device__ __forceinline__ int snake_pos(int r, int cta, int ncta) {
    return r * ncta + ((r & 1) ? ncta - 1 - cta : cta);
}
// the position after pos = snake_pos(r, cta, ncta)
__device__ __forceinline__ int snake_next(int pos, int cta, int ncta) {
    return snake_pos(pos / ncta + 1, cta, ncta);
}

}  // namespace
}  // namespace pk
