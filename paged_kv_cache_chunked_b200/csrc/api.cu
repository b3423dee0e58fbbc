// Host side of the C ABI: argument checks, pool descriptors (with the TMA
// tensor maps the attention kernel reads through), dispatch to the kernels.
#include "pk_internal.h"

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

namespace pk {

static thread_local char g_err[512];

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(PK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

bool force_generic() {
    const char *e = getenv("PK_FORCE_GENERIC");
    return e && e[0] == '1';
}

}  // namespace

// 2-D view of a pool: rows = num_blocks * n_kv_heads * block_size token rows of
// head_dim bf16 each; box = 64 columns (128 bytes, the swizzle span) x box_rows.
int encode_pool_map(CUtensorMap *map, void *base, const pk_pool *p, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PK_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[2] = {(cuuint64_t)p->head_dim,
                                (cuuint64_t)p->num_blocks * p->n_kv_heads * p->block_size};
    const cuuint64_t strides[1] = {(cuuint64_t)p->head_dim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PK_OK;
}

// 3-D view of the same rows: x = column within a 64-column panel, y = row, z =
// panel (stride 128 bytes).  A box {64, box_rows, head_dim / 64} lands in shared
// memory as head_dim / 64 consecutive panels of box_rows 128-byte rows, the
// layout of box_rows-row 2-D boxes placed panel after panel.
int encode_pool_map3(CUtensorMap *map, void *base, const pk_pool *p, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(PK_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    const cuuint64_t dims[3] = {64, (cuuint64_t)p->num_blocks * p->n_kv_heads * p->block_size,
                                (cuuint64_t)p->head_dim / 64};
    const cuuint64_t strides[2] = {(cuuint64_t)p->head_dim * 2, 128};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)p->head_dim / 64};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PK_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed (%d)", (int)r);
    return PK_OK;
}

}  // namespace pk

using namespace pk;

extern "C" {

const char *pk_last_error(void) { return g_err; }

const char *pk_version(void) { return "paged_kv 0.1 (sm_100a)"; }

int pk_pool_create(int num_blocks, int block_size, int n_kv_heads, int head_dim, int dtype,
                   void *k_base, void *v_base, pk_pool **out) {
    g_err[0] = 0;
    if (!out) return fail(PK_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (num_blocks < 1 || block_size < 1 || n_kv_heads < 1 || head_dim < 1)
        return fail(PK_ERR_INVALID_ARG, "pool geometry must be positive");
    if (head_dim > kMaxHeadDim) return fail(PK_ERR_UNSUPPORTED, "head_dim %d > %d", head_dim, kMaxHeadDim);
    if (dtype != PK_F32 && dtype != PK_BF16) return fail(PK_ERR_UNSUPPORTED, "dtype %d", dtype);
    if (!k_base || !v_base) return fail(PK_ERR_INVALID_ARG, "pool base pointer is NULL");
    if (!aligned(k_base, 16) || !aligned(v_base, 16))
        return fail(PK_ERR_INVALID_ARG, "pool bases must be 16-byte aligned");

    pk_pool *p = new (std::nothrow) pk_pool();
    if (!p) return fail(PK_ERR_INVALID_ARG, "out of host memory");
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->n_kv_heads = n_kv_heads;
    p->head_dim = head_dim;
    p->dtype = dtype;
    p->k_base = k_base;
    p->v_base = v_base;
    cudaError_t e = cudaGetDevice(&p->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device);
    if (e == cudaSuccess) e = cudaMalloc(&p->d_err, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(p->d_err, 0, sizeof(int));
    if (e != cudaSuccess) {
        if (p->d_err) cudaFree(p->d_err);
        delete p;
        return cuda_fail(e, "pool create");
    }
    const long long rows = (long long)num_blocks * n_kv_heads * block_size;
    p->tc_path = dtype == PK_BF16 && (head_dim == 64 || head_dim == 128 || head_dim == 256) &&
                 block_size % 8 == 0 && n_kv_heads <= kMaxTcKvHeads && rows < (1LL << 31) &&
                 !force_generic();
    if (p->tc_path) {
        // 16-token tiles of one (block, kv head): one 3-D box brings all head-dim
        // panels when a tile lies in one block (block_size a multiple of 16);
        // else two 2-D boxes of 8 rows per panel
        const int box = block_size % kTile == 0 ? kTile : 8;
        p->tile_map3d = box == kTile;
        int rc = p->tile_map3d ? encode_pool_map3(&p->tmap_k, k_base, p, box)
                               : encode_pool_map(&p->tmap_k, k_base, p, box);
        if (rc == PK_OK)
            rc = p->tile_map3d ? encode_pool_map3(&p->tmap_v, v_base, p, box)
                               : encode_pool_map(&p->tmap_v, v_base, p, box);
        if (rc == PK_OK) rc = tc_prepare_pool(p);
        if (rc != PK_OK) {
            cudaFree(p->d_err);
            delete p;
            return rc;
        }
    }
    *out = p;
    return PK_OK;
}

int pk_pool_destroy(pk_pool *pool) {
    if (!pool) return PK_OK;
    int dev = -1;
    cudaGetDevice(&dev);
    if (dev != pool->device) cudaSetDevice(pool->device);
    cudaError_t e = cudaFree(pool->d_err);
    if (dev >= 0 && dev != pool->device) cudaSetDevice(dev);
    delete pool;
    return e == cudaSuccess ? PK_OK : cuda_fail(e, "pool destroy");
}

int pk_pool_paths(const pk_pool *pool, int *paths_out) {
    if (!pool || !paths_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    int f = 0;
    if (pool->tc_path) {
        f |= PK_PATH_TENSOR_CORE;
        if (pool->blk_ok) f |= PK_PATH_DECODE_BLOCKS;
        if (pool->umma_ok || pool->umma256_ok) f |= PK_PATH_CHUNK_TCGEN05;
    }
    *paths_out = f;
    return PK_OK;
}

int pk_check_device_errors(const pk_pool *pool, pk_stream_t stream, int *code_out) {
    if (!pool || !code_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    int h = 0;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(&h, pool->d_err, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(pool->d_err, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    *code_out = h;
    return PK_OK;
}

int pk_paged_kv_append(const pk_pool *pool, const void *k, const void *v,
                       const int64_t *slot_mapping, int num_tokens, pk_stream_t stream) {
    if (!pool) return fail(PK_ERR_INVALID_ARG, "pool is NULL");
    if (num_tokens < 0) return fail(PK_ERR_INVALID_ARG, "num_tokens < 0");
    if (num_tokens > 0 && (!k || !v || !slot_mapping))
        return fail(PK_ERR_INVALID_ARG, "NULL k, v or slot_mapping");
    if (!aligned(slot_mapping, 8)) return fail(PK_ERR_INVALID_ARG, "slot_mapping misaligned");
    return launch_kv_append(pool, k, v, slot_mapping, num_tokens, (cudaStream_t)stream);
}

int pk_block_copy(const pk_pool *pool, const int32_t *src_dst_pairs, int n_pairs,
                  pk_stream_t stream) {
    if (!pool) return fail(PK_ERR_INVALID_ARG, "pool is NULL");
    if (n_pairs < 0) return fail(PK_ERR_INVALID_ARG, "n_pairs < 0");
    if (n_pairs > 0 && !src_dst_pairs) return fail(PK_ERR_INVALID_ARG, "NULL pairs");
    return launch_block_copy(pool, src_dst_pairs, n_pairs, (cudaStream_t)stream);
}

int pk_swap_blocks(const pk_pool *pool, void *host_k, void *host_v, int num_host_blocks,
                   const int32_t *pairs, int n_pairs, int to_host, pk_stream_t stream) {
    if (!pool) return fail(PK_ERR_INVALID_ARG, "pool is NULL");
    if (n_pairs < 0 || num_host_blocks < 0) return fail(PK_ERR_INVALID_ARG, "negative count");
    if (n_pairs == 0) return PK_OK;
    if (!pairs || !host_k || !host_v) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    // the kernel reaches the host pool through its device mapping: only
    // page-locked host memory with one is accepted
    void *view[2] = {nullptr, nullptr};
    void *host[2] = {host_k, host_v};
    for (int i = 0; i < 2; ++i) {
        cudaPointerAttributes at;
        const cudaError_t e = cudaPointerGetAttributes(&at, host[i]);
        if (e != cudaSuccess) return cuda_fail(e, "host pool pointer attributes");
        if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr)
            return fail(PK_ERR_INVALID_ARG, "host pool is not page-locked host memory mapped for the device");
        view[i] = at.devicePointer;
    }
    return launch_swap_blocks(pool, view[0], view[1], num_host_blocks, pairs, n_pairs, to_host != 0,
                              (cudaStream_t)stream);
}

int pk_attention_workspace_size(const pk_pool *pool, int num_seqs, int num_tokens,
                                int n_q_heads, int max_blocks_per_seq, size_t *bytes_out) {
    if (!pool || !bytes_out) return fail(PK_ERR_INVALID_ARG, "NULL argument");
    if (num_seqs < 0 || num_tokens < 0 || n_q_heads < 1 || max_blocks_per_seq < 0 ||
        n_q_heads % pool->n_kv_heads != 0)
        return fail(PK_ERR_INVALID_ARG, "bad batch shape");
    *bytes_out = pool->tc_path
                     ? tc_workspace_bytes(pool, num_seqs, num_tokens, n_q_heads, max_blocks_per_seq)
                     : 256;
    return PK_OK;
}

}  // extern "C"

namespace {

// Checks and launch shared by the two attention entry points; append: the
// query rows' own K/V (k_new, v_new) are stored first.
int attention_call(const pk_pool *pool, const void *q, bool append, const void *k_new, const void *v_new,
                   void *out,
                   const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
                   const int32_t *query_start_lens, int num_seqs, int num_tokens, int n_q_heads, float scale,
                   void *workspace, size_t workspace_bytes, pk_stream_t stream) {
    if (!pool) return fail(PK_ERR_INVALID_ARG, "pool is NULL");
    if (num_seqs < 0 || num_tokens < num_seqs || n_q_heads < 1 || max_blocks_per_seq < 1)
        return fail(PK_ERR_INVALID_ARG, "bad batch shape (num_seqs %d, num_tokens %d)", num_seqs,
                    num_tokens);
    if (n_q_heads % pool->n_kv_heads != 0)
        return fail(PK_ERR_INVALID_ARG, "n_q_heads %d not a multiple of n_kv_heads %d", n_q_heads,
                    pool->n_kv_heads);
    if (num_seqs == 0) return PK_OK;
    if (!q || !out || !block_tables || !context_lens || !query_start_lens)
        return fail(PK_ERR_INVALID_ARG, "NULL pointer argument");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(block_tables, 4) ||
        !aligned(context_lens, 4) || !aligned(query_start_lens, 4))
        return fail(PK_ERR_INVALID_ARG, "misaligned pointer argument");
    if (append && (!k_new || !v_new)) return fail(PK_ERR_INVALID_ARG, "NULL k or v");
    if (append && (!aligned(k_new, 16) || !aligned(v_new, 16)))
        return fail(PK_ERR_INVALID_ARG, "misaligned k or v");
    if (!(scale > 0.f) || scale != scale) return fail(PK_ERR_INVALID_ARG, "scale must be > 0");
    AttnArgs a{q, out, block_tables, max_blocks_per_seq, context_lens, query_start_lens,
               num_seqs, num_tokens, n_q_heads, scale, workspace, workspace_bytes, k_new, v_new};
    if (pool->tc_path) return launch_attention_tc(pool, a, (cudaStream_t)stream);
    if (append) {
        const int rc = launch_kv_append_at_positions(pool, a, (cudaStream_t)stream);
        if (rc != PK_OK) return rc;
    }
    return launch_attention_generic(pool, a, (cudaStream_t)stream);
}

}  // namespace

extern "C" {

int pk_paged_attention(const pk_pool *pool, const void *q, void *out,
                       const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, const int32_t *query_start_lens,
                       int num_seqs, int num_tokens, int n_q_heads, float scale,
                       void *workspace, size_t workspace_bytes, pk_stream_t stream) {
    return attention_call(pool, q, false, nullptr, nullptr, out, block_tables, max_blocks_per_seq, context_lens,
                          query_start_lens, num_seqs, num_tokens, n_q_heads, scale, workspace,
                          workspace_bytes, stream);
}

int pk_paged_attention_append(const pk_pool *pool, const void *q, const void *k, const void *v, void *out,
                              const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *context_lens, const int32_t *query_start_lens,
                              int num_seqs, int num_tokens, int n_q_heads, float scale,
                              void *workspace, size_t workspace_bytes, pk_stream_t stream) {
    return attention_call(pool, q, true, k, v, out, block_tables, max_blocks_per_seq, context_lens,
                          query_start_lens, num_seqs, num_tokens, n_q_heads, scale, workspace,
                          workspace_bytes, stream);
}

}  // extern "C"
