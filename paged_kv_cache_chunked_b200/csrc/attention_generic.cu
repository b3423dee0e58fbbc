// General paged attention kernel: any head_dim <= 256, any block size, fp32
// or bf16 storage, fp32 arithmetic.  It serves the float32 pools (where the
// tensor cores would have to round inputs to tf32) and geometries outside the
// tensor-core kernel's tiling.
//
// What it computes ["PagedAttention & Continuous Batching" (study notes),
// "Block tables": the kernel gathers K/V through the block table; "Batching
// and PagedAttention", "Continuous batching": chunked prefill]: for query
// token i of sequence b (position p = c_b - q_b + i) and q head h, softmax
// attention over keys 0..p of kv head h / (Hq / Hkv), each key read from
// block table_b[j / bs], slot j % bs.
//
// One warp per (query token, q head).  The lanes split head_dim; each key's
// dot product is a warp reduction, followed by an online-softmax update
// (running max, running sum, rescaled accumulator) in fp32 registers.
#include "pk_internal.h"

#include <cuda_bf16.h>

namespace pk {
namespace {

constexpr int kWarps = 4;
constexpr int kMaxPerLane = kMaxHeadDim / 32;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f32(float v, float *dst) { *dst = v; }
__device__ __forceinline__ void from_f32(float v, __nv_bfloat16 *dst) { *dst = __float2bfloat16_rn(v); }

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
attention_generic_kernel(const T *__restrict__ q, T *__restrict__ out, const T *__restrict__ kp,
                         const T *__restrict__ vp, const int32_t *__restrict__ tables,
                         int max_blocks, const int32_t *__restrict__ ctx_lens,
                         const int32_t *__restrict__ qsl, int num_seqs, int num_tokens,
                         int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                         int num_blocks, float scale, int *err) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (row >= (int64_t)num_tokens * n_q_heads) return;
    const int t = (int)(row / n_q_heads);
    const int h = (int)(row % n_q_heads);

    // sequence of token t: last b with qsl[b] <= t
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(qsl + mid) <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int c = __ldg(ctx_lens + b);
    const int qlen = __ldg(qsl + b + 1) - __ldg(qsl + b);
    const int pos = c - qlen + (t - __ldg(qsl + b));
    if (qlen < 1 || c < qlen || (c + block_size - 1) / block_size > max_blocks || pos < 0) {
        if (lane == 0) record_error(err, PK_ERR_BAD_INDEX);
        return;
    }
    const int kvh = h / (n_q_heads / n_kv_heads);
    const int32_t *table = tables + (int64_t)b * max_blocks;

    float qv[kMaxPerLane], acc[kMaxPerLane];
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
        const int e = lane + 32 * k;
        qv[k] = e < head_dim ? to_f32(q[row * head_dim + e]) : 0.f;
        acc[k] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    int cur_blk = -1;
    const T *kbase = nullptr, *vbase = nullptr;
    for (int j = 0; j <= pos; ++j) {
        const int lb = j / block_size;
        if (lb != cur_blk) {
            cur_blk = lb;
            int phys = __ldg(table + lb);
            if (phys < 0 || phys >= num_blocks) {
                if (lane == 0) record_error(err, PK_ERR_BAD_INDEX);
                phys = 0;
            }
            const int64_t off = ((int64_t)phys * n_kv_heads + kvh) * block_size * head_dim;
            kbase = kp + off;
            vbase = vp + off;
        }
        const int slot = j % block_size;
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < kMaxPerLane; ++k) {
            const int e = lane + 32 * k;
            if (e < head_dim) s += qv[k] * to_f32(kbase[slot * head_dim + e]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        s *= scale;
        const float m_new = fmaxf(m, s);
        const float alpha = expf(m - m_new);   // m = -inf on the first key: alpha = 0
        const float pj = expf(s - m_new);
        l = l * alpha + pj;
#pragma unroll
        for (int k = 0; k < kMaxPerLane; ++k) {
            const int e = lane + 32 * k;
            const float vv = e < head_dim ? to_f32(vbase[slot * head_dim + e]) : 0.f;
            acc[k] = acc[k] * alpha + pj * vv;
        }
        m = m_new;
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int k = 0; k < kMaxPerLane; ++k) {
        const int e = lane + 32 * k;
        if (e < head_dim) from_f32(acc[k] * inv, out + row * head_dim + e);
    }
}

}  // namespace

int launch_attention_generic(const pk_pool *p, const AttnArgs &a, cudaStream_t st) {
    const int64_t rows = (int64_t)a.num_tokens * a.n_q_heads;
    if (rows == 0) return PK_OK;
    const int64_t grid = (rows + kWarps - 1) / kWarps;
    if (grid > 0x7fffffff) return fail(PK_ERR_INVALID_ARG, "too many query rows");
    if (p->dtype == PK_BF16)
        attention_generic_kernel<__nv_bfloat16><<<(unsigned)grid, kWarps * 32, 0, st>>>(
            (const __nv_bfloat16 *)a.q, (__nv_bfloat16 *)a.out, (const __nv_bfloat16 *)p->k_base,
            (const __nv_bfloat16 *)p->v_base, a.block_tables, a.max_blocks_per_seq,
            a.context_lens, a.query_start_lens, a.num_seqs, a.num_tokens, a.n_q_heads,
            p->n_kv_heads, p->head_dim, p->block_size, p->num_blocks, a.scale, p->d_err);
    else
        attention_generic_kernel<float><<<(unsigned)grid, kWarps * 32, 0, st>>>(
            (const float *)a.q, (float *)a.out, (const float *)p->k_base,
            (const float *)p->v_base, a.block_tables, a.max_blocks_per_seq, a.context_lens,
            a.query_start_lens, a.num_seqs, a.num_tokens, a.n_q_heads, p->n_kv_heads,
            p->head_dim, p->block_size, p->num_blocks, a.scale, p->d_err);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "generic attention launch");
}

}  // namespace pk
