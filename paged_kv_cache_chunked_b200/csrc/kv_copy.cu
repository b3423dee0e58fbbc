// Slot-mapped KV append and whole-block copy (copy-on-write).
//
// Append ["PagedAttention & Continuous Batching" (study notes), "Flow" step 4:
// new tokens' K/V go into the blocks their table maps them to]: token t's K
// and V rows (all kv heads) are stored at slot slot_mapping[t] = block *
// block_size + offset; negative slots are skipped.
// Block copy [same page, "Copy-on-write": a write into a shared block takes a
// fresh block and copies it first]: block dst receives all of block src, K
// and V.
//
// Both are pure data movement, bound by HBM bandwidth: each thread moves
// 16-byte vectors with streaming loads/stores, consecutive threads touch
// consecutive 16-byte chunks of one (block, head) row so every warp access is
// a full 512-byte coalesced segment.
#include "pk_internal.h"

namespace pk {
namespace {

// Each kernel here is launched as a programmatic dependent of the previous
// kernel on the stream (launch_dependent).  It lets its own dependent (the next
// copy, or the attention kernel, whose plan reads no pool rows) start launching
// at once, then waits for the previous grid to finish, and its writes to be
// visible, before it touches any memory: stream order as seen by memory is
// unchanged, but the launch no longer waits for the previous grid's last CTA.
__device__ __forceinline__ void pdl_prologue() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
}


// One warp per token: the token's slot is read and split into (block, offset)
// once, then the lanes move the token's K and V rows of all kv heads
// (n_kv_heads * row_chunks 16-byte chunks each), four chunks of K and four of V
// a lane, all loads issued before the first store.  Consecutive lanes touch
// consecutive chunks of one (block, head) row, so every warp access is a
// contiguous 512-byte run.  Grid-stride over the tokens.
constexpr int kAppendUnroll = 4;
__global__ void kv_append_vec16(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                uint4 *__restrict__ kp, uint4 *__restrict__ vp,
                                const int64_t *__restrict__ slots, int num_tokens, int n_kv_heads,
                                int block_size, int row_chunks, int64_t num_slots,
                                int *err) {
    pdl_prologue();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    const int per_side = n_kv_heads * row_chunks;  // chunks of one token's K (or V)
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < num_tokens; t += warps) {
        const int64_t slot = __ldg(slots + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (lane == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int off = (int)(slot - blk * block_size);
        // chunk c = h * row_chunks + e of the token goes to ((blk * Hkv + h) * bs + off) * row_chunks + e
        const int64_t base = (blk * n_kv_heads * block_size + off) * row_chunks;
        const int64_t head_stride = (int64_t)block_size * row_chunks;
        const uint4 *ks = k + (int64_t)t * per_side, *vs = v + (int64_t)t * per_side;
        for (int c0 = 0; c0 < per_side; c0 += 32 * kAppendUnroll) {
            uint4 a[kAppendUnroll], b[kAppendUnroll];
#pragma unroll
            for (int u = 0; u < kAppendUnroll; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < per_side) {
                    a[u] = __ldcs(ks + c);
                    b[u] = __ldcs(vs + c);
                }
            }
#pragma unroll
            for (int u = 0; u < kAppendUnroll; ++u) {
                const int c = c0 + u * 32 + lane;
                if (c < per_side) {
                    const int h = c / row_chunks;
                    const int64_t dst = base + h * head_stride + (c - h * row_chunks);
                    __stcs(kp + dst, a[u]);
                    __stcs(vp + dst, b[u]);
                }
            }
        }
    }
}

// The query rows' K/V of an attention call stored at their positions: token t
// of sequence b (t = qsl[b] + i) sits at position ctx[b] - (qsl[b + 1] - qsl[b])
// + i, in block tables[b][pos / bs] at offset pos % bs.  One warp per token;
// the sequence is found by a binary search over the query offsets.  A row is
// row_elems elements of T (16-byte vectors when the row allows, else scalars).
template <typename T>
__global__ void kv_append_at_positions(const T *__restrict__ k, const T *__restrict__ v, T *kp, T *vp,
                                       const int32_t *__restrict__ tables, int max_blocks,
                                       const int32_t *__restrict__ ctx, const int32_t *__restrict__ qsl,
                                       int num_seqs, int num_tokens, int n_kv_heads, int block_size,
                                       int row_elems, int num_blocks, int *err) {
    pdl_prologue();
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    const int per_side = n_kv_heads * row_elems;
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < num_tokens; t += warps) {
        int lo = 0, hi = num_seqs - 1;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (__ldg(qsl + mid + 1) > t) hi = mid;
            else lo = mid + 1;
        }
        const int b = lo;
        const int s0 = __ldg(qsl + b), s1 = __ldg(qsl + b + 1), c = __ldg(ctx + b);
        const int pos = c - (s1 - s0) + (t - s0);
        if (t < s0 || t >= s1 || pos < 0 || pos >= max_blocks * block_size) {
            if (lane == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const int blk = __ldg(tables + (int64_t)b * max_blocks + pos / block_size);
        if (blk < 0 || blk >= num_blocks) {
            if (lane == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const int off = pos % block_size;
        const T *ks = k + (int64_t)t * per_side, *vs = v + (int64_t)t * per_side;
        for (int c2 = lane; c2 < per_side; c2 += 32) {
            const int h = c2 / row_elems;
            const int64_t dst = (((int64_t)blk * n_kv_heads + h) * block_size + off) * row_elems + (c2 - h * row_elems);
            kp[dst] = ks[c2];
            vp[dst] = vs[c2];
        }
    }
}

// Element-wise fallback for rows that are not a multiple of 16 bytes.
template <typename T>
__global__ void kv_append_scalar(const T *__restrict__ k, const T *__restrict__ v, T *kp, T *vp,
                                 const int64_t *__restrict__ slots, int num_tokens,
                                 int n_kv_heads, int block_size, int head_dim,
                                 int64_t num_slots, int *err) {
    pdl_prologue();
    const int64_t per_side = (int64_t)num_tokens * n_kv_heads * head_dim;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < 2 * per_side;
         i += (int64_t)gridDim.x * blockDim.x) {
        const bool is_v = i >= per_side;
        const int64_t j = is_v ? i - per_side : i;
        const int e = (int)(j % head_dim);
        const int64_t th = j / head_dim;
        const int h = (int)(th % n_kv_heads);
        const int64_t t = th / n_kv_heads;
        const int64_t slot = slots[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const int64_t dst = (((slot / block_size) * n_kv_heads + h) * block_size +
                             slot % block_size) * head_dim + e;
        (is_v ? vp : kp)[dst] = (is_v ? v : k)[j];
    }
}

// One CTA per (pair, K or V); the block's bytes are copied as 16-byte vectors.
__global__ void block_copy_vec16(uint4 *kp, uint4 *vp, const int32_t *__restrict__ pairs,
                                 int n_pairs, int64_t block_chunks, int num_blocks, int *err) {
    pdl_prologue();
    for (int64_t w = blockIdx.x; w < 2LL * n_pairs; w += gridDim.x) {
        const int pr = (int)(w >> 1);
        uint4 *pool = (w & 1) ? vp : kp;
        const int src = __ldg(pairs + 2 * pr);
        const int dst = __ldg(pairs + 2 * pr + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (threadIdx.x == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const uint4 *s = pool + (int64_t)src * block_chunks;
        uint4 *d = pool + (int64_t)dst * block_chunks;
        // unrolled by 4 so that each thread keeps several loads in flight
        int64_t i = threadIdx.x;
        for (; i + 3 * blockDim.x < block_chunks; i += 4 * blockDim.x) {
            uint4 a = __ldcs(s + i), b = __ldcs(s + i + blockDim.x);
            uint4 c = __ldcs(s + i + 2 * blockDim.x), e = __ldcs(s + i + 3 * blockDim.x);
            __stcs(d + i, a);
            __stcs(d + i + blockDim.x, b);
            __stcs(d + i + 2 * blockDim.x, c);
            __stcs(d + i + 3 * blockDim.x, e);
        }
        for (; i < block_chunks; i += blockDim.x) __stcs(d + i, __ldcs(s + i));
    }
}

template <typename T>
__global__ void block_copy_scalar(T *kp, T *vp, const int32_t *__restrict__ pairs, int n_pairs,
                                  int64_t block_elems, int num_blocks, int *err) {
    pdl_prologue();
    for (int64_t w = blockIdx.x; w < 2LL * n_pairs; w += gridDim.x) {
        const int pr = (int)(w >> 1);
        T *pool = (w & 1) ? vp : kp;
        const int src = pairs[2 * pr], dst = pairs[2 * pr + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (threadIdx.x == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        for (int64_t i = threadIdx.x; i < block_elems; i += blockDim.x)
            pool[(int64_t)dst * block_elems + i] = pool[(int64_t)src * block_elems + i];
    }
}

// Whole blocks between two pools of the same block geometry (the device pool
// and a host pool, in either direction): CTA work item w copies K (w even) or
// V (w odd) of pair w / 2, a = source block, b = destination block.  The host
// side is read or written over the host link through its device mapping.
template <typename T, int UNROLL>
__global__ void swap_copy(const T *__restrict__ sk, const T *__restrict__ sv, T *dk, T *dv,
                          const int32_t *__restrict__ pairs, int n_pairs, int64_t block_chunks,
                          int n_src, int n_dst, int *err) {
    pdl_prologue();
    for (int64_t w = blockIdx.x; w < 2LL * n_pairs; w += gridDim.x) {
        const int pr = (int)(w >> 1);
        const int a = __ldg(pairs + 2 * pr), b = __ldg(pairs + 2 * pr + 1);
        if (a < 0 || a >= n_src || b < 0 || b >= n_dst) {
            if (threadIdx.x == 0) record_error(err, PK_ERR_BAD_INDEX);
            continue;
        }
        const T *src = ((w & 1) ? sv : sk) + (int64_t)a * block_chunks;
        T *dst = ((w & 1) ? dv : dk) + (int64_t)b * block_chunks;
        int64_t i = threadIdx.x;
        // several loads in flight per thread: the host link's latency is long
        for (; i + (UNROLL - 1) * blockDim.x < block_chunks; i += UNROLL * blockDim.x) {
            T r[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) r[u] = src[i + u * blockDim.x];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) dst[i + u * blockDim.x] = r[u];
        }
        for (; i < block_chunks; i += blockDim.x) dst[i] = src[i];
    }
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

int grid_for(int64_t work, int threads, int sm_count) {
    int64_t g = (work + threads - 1) / threads;
    int64_t cap = (int64_t)sm_count * 16;
    if (g > cap) g = cap;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

int launch_kv_append(const pk_pool *p, const void *k, const void *v, const int64_t *slots,
                     int num_tokens, cudaStream_t st) {
    if (num_tokens == 0) return PK_OK;
    const int elt = p->dtype == PK_BF16 ? 2 : 4;
    const int64_t row_bytes = (int64_t)p->head_dim * elt;
    const int64_t num_slots = (int64_t)p->num_blocks * p->block_size;
    cudaError_t e;
    if (row_bytes % 16 == 0 && aligned16(k) && aligned16(v)) {
        const int row_chunks = (int)(row_bytes / 16);
        // one warp per token, eight warps a CTA
        e = launch_dependent(kv_append_vec16, dim3(grid_for(32LL * num_tokens, 256, p->sm_count)), 256, 0, st, (const uint4 *)k,
                       (const uint4 *)v, (uint4 *)p->k_base, (uint4 *)p->v_base, slots, num_tokens,
                       p->n_kv_heads, p->block_size, row_chunks, num_slots, p->d_err);
    } else {
        const int64_t work = 2LL * num_tokens * p->n_kv_heads * p->head_dim;
        const int grid = grid_for(work, 256, p->sm_count);
        if (p->dtype == PK_BF16)
            e = launch_dependent(kv_append_scalar<uint16_t>, dim3(grid), 256, 0, st, (const uint16_t *)k,
                           (const uint16_t *)v, (uint16_t *)p->k_base, (uint16_t *)p->v_base, slots,
                           num_tokens, p->n_kv_heads, p->block_size, p->head_dim, num_slots, p->d_err);
        else
            e = launch_dependent(kv_append_scalar<float>, dim3(grid), 256, 0, st, (const float *)k, (const float *)v,
                           (float *)p->k_base, (float *)p->v_base, slots, num_tokens, p->n_kv_heads,
                           p->block_size, p->head_dim, num_slots, p->d_err);
    }
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "kv append launch");
}

int launch_kv_append_at_positions(const pk_pool *p, const AttnArgs &a, cudaStream_t st) {
    if (a.num_tokens == 0 || a.num_seqs == 0) return PK_OK;
    const int elt = p->dtype == PK_BF16 ? 2 : 4;
    const int64_t row_bytes = (int64_t)p->head_dim * elt;
    const int grid = grid_for(32LL * a.num_tokens, 256, p->sm_count);  // one warp per token
    cudaError_t e;
    if (row_bytes % 16 == 0 && aligned16(a.k_new) && aligned16(a.v_new))
        e = launch_dependent(kv_append_at_positions<uint4>, dim3(grid), 256, 0, st, (const uint4 *)a.k_new,
                             (const uint4 *)a.v_new, (uint4 *)p->k_base, (uint4 *)p->v_base, a.block_tables,
                             a.max_blocks_per_seq, a.context_lens, a.query_start_lens, a.num_seqs, a.num_tokens,
                             p->n_kv_heads, p->block_size, (int)(row_bytes / 16), p->num_blocks, p->d_err);
    else if (p->dtype == PK_BF16)
        e = launch_dependent(kv_append_at_positions<uint16_t>, dim3(grid), 256, 0, st, (const uint16_t *)a.k_new,
                             (const uint16_t *)a.v_new, (uint16_t *)p->k_base, (uint16_t *)p->v_base,
                             a.block_tables, a.max_blocks_per_seq, a.context_lens, a.query_start_lens, a.num_seqs,
                             a.num_tokens, p->n_kv_heads, p->block_size, p->head_dim, p->num_blocks, p->d_err);
    else
        e = launch_dependent(kv_append_at_positions<float>, dim3(grid), 256, 0, st, (const float *)a.k_new,
                             (const float *)a.v_new, (float *)p->k_base, (float *)p->v_base, a.block_tables,
                             a.max_blocks_per_seq, a.context_lens, a.query_start_lens, a.num_seqs, a.num_tokens,
                             p->n_kv_heads, p->block_size, p->head_dim, p->num_blocks, p->d_err);
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "kv append at positions launch");
}

int launch_swap_blocks(const pk_pool *p, void *host_k, void *host_v, int num_host_blocks,
                       const int32_t *pairs, int n_pairs, bool to_host, cudaStream_t st) {
    if (n_pairs == 0) return PK_OK;
    const int elt = p->dtype == PK_BF16 ? 2 : 4;
    const int64_t block_elems = (int64_t)p->n_kv_heads * p->block_size * p->head_dim;
    const int64_t block_bytes = block_elems * elt;
    void *sk = to_host ? p->k_base : host_k, *sv = to_host ? p->v_base : host_v;
    void *dk = to_host ? host_k : p->k_base, *dv = to_host ? host_v : p->v_base;
    const int n_src = to_host ? p->num_blocks : num_host_blocks;
    const int n_dst = to_host ? num_host_blocks : p->num_blocks;
    const int64_t ctas = 2LL * n_pairs;
    const int grid = (int)(ctas < (int64_t)p->sm_count * 32 ? ctas : (int64_t)p->sm_count * 32);
    cudaError_t e;
    if (block_bytes % 16 == 0 && aligned16(sk) && aligned16(sv) && aligned16(dk) && aligned16(dv))
        e = launch_dependent(swap_copy<uint4, 4>, dim3(grid), 256, 0, st, (const uint4 *)sk, (const uint4 *)sv,
                       (uint4 *)dk, (uint4 *)dv, pairs, n_pairs, block_bytes / 16, n_src, n_dst,
                       p->d_err);
    else if (p->dtype == PK_BF16)
        e = launch_dependent(swap_copy<uint16_t, 4>, dim3(grid), 256, 0, st, (const uint16_t *)sk,
                       (const uint16_t *)sv, (uint16_t *)dk, (uint16_t *)dv, pairs, n_pairs,
                       block_elems, n_src, n_dst, p->d_err);
    else
        e = launch_dependent(swap_copy<float, 4>, dim3(grid), 256, 0, st, (const float *)sk, (const float *)sv,
                       (float *)dk, (float *)dv, pairs, n_pairs, block_elems, n_src, n_dst, p->d_err);
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "block swap launch");
}

int launch_block_copy(const pk_pool *p, const int32_t *pairs, int n_pairs, cudaStream_t st) {
    if (n_pairs == 0) return PK_OK;
    const int elt = p->dtype == PK_BF16 ? 2 : 4;
    const int64_t block_elems = (int64_t)p->n_kv_heads * p->block_size * p->head_dim;
    const int64_t block_bytes = block_elems * elt;
    const int64_t ctas = 2LL * n_pairs;
    const int grid = (int)(ctas < (int64_t)p->sm_count * 32 ? ctas : (int64_t)p->sm_count * 32);
    cudaError_t e;
    if (block_bytes % 16 == 0)
        e = launch_dependent(block_copy_vec16, dim3(grid), 256, 0, st, (uint4 *)p->k_base, (uint4 *)p->v_base, pairs,
                       n_pairs, block_bytes / 16, p->num_blocks, p->d_err);
    else if (p->dtype == PK_BF16)
        e = launch_dependent(block_copy_scalar<uint16_t>, dim3(grid), 256, 0, st, (uint16_t *)p->k_base,
                       (uint16_t *)p->v_base, pairs, n_pairs, block_elems, p->num_blocks, p->d_err);
    else
        e = launch_dependent(block_copy_scalar<float>, dim3(grid), 256, 0, st, (float *)p->k_base,
                       (float *)p->v_base, pairs, n_pairs, block_elems, p->num_blocks, p->d_err);
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "block copy launch");
}

}  // namespace pk
