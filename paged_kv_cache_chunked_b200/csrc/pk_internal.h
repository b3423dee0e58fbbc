// Internal declarations of the paged KV library (not part of the C ABI).
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver entry point is fetched at run time)
#include <cuda_runtime.h>
#include <stdint.h>

#include "paged_kv.h"

// Pool descriptor behind the opaque pk_pool handle.
struct pk_pool {
    int num_blocks;
    int block_size;
    int n_kv_heads;
    int head_dim;
    int dtype;  // PK_F32 / PK_BF16
    void *k_base;
    void *v_base;
    int *d_err;       // device error word (first recorded PK_ERR_* code)
    int device;
    int sm_count;
    bool tc_path;       // tensor-core + TMA attention applies to this geometry
    int tc_ctas;        // resident CTAs of the decode attention kernel (whole GPU)
    int tc_ctas_chunk;  // resident CTAs of the chunk attention kernel (whole GPU)
    bool tile_map3d;    // tmap_k / tmap_v are 3-D (16-row boxes of all panels), else 2-D (8 rows)
    bool umma_ok;       // the tcgen05 chunk kernel serves this geometry (head dim 64 / 128)
    bool umma256_ok;    // the head-dim-256 tcgen05 chunk kernel serves it
    bool blk_ok;        // the block-streaming decode kernel serves this geometry
    int blk_hs, blk_nbs;  // its kv heads and blocks per pipeline stage
    int blk_smem_max;     // its largest dynamic shared memory per launch
    alignas(64) CUtensorMap tmap_k;
    alignas(64) CUtensorMap tmap_v;
    alignas(64) CUtensorMap tmap_kb;  // 3-D boxes of blk_hs * block_size rows, all panels
    alignas(64) CUtensorMap tmap_vb;
    alignas(64) CUtensorMap tmap_k2;  // 2-D, 16-row boxes: K tiles of the tcgen05 chunk kernel
};

namespace pk {

// Sets the thread-local error message; returns `code`.
int fail(int code, const char *fmt, ...);
int cuda_fail(cudaError_t e, const char *what);

// Records `code` in the device error word unless an earlier code is there.
__device__ __forceinline__ void record_error(int *err, int code) {
    if (err) atomicCAS(err, 0, code);
}

constexpr int kMaxHeadDim = 256;
constexpr int kTile = 16;        // tokens per KV tile and rows per query tile
constexpr int kMaxSeqsPerLaunch = 512;  // window of sequences per kernel launch
// Largest n_kv_heads of the tensor-core path: the workspace keeps one split-K
// arrival counter per (sequence of a launch window, kv head) in a region of
// fixed size, so that every pool finds its counters at the same offsets.
constexpr int kMaxTcKvHeads = 64;

// Launches kernel as a programmatic dependent of the previous kernel on the
// stream: it may start while that kernel drains, so it must execute
// griddepcontrol.wait before it reads what earlier work on the stream wrote
// (or writes what that work reads).
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, int threads, size_t smem, cudaStream_t st,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, ((KArgs)args)...);
}

// ---- launchers (each returns PK_OK or an error code) ---------------------
int launch_kv_append(const pk_pool *p, const void *k, const void *v, const int64_t *slots,
                     int num_tokens, cudaStream_t st);
int launch_block_copy(const pk_pool *p, const int32_t *pairs, int n_pairs, cudaStream_t st);
int launch_swap_blocks(const pk_pool *p, void *host_k, void *host_v, int num_host_blocks,
                       const int32_t *pairs, int n_pairs, bool to_host, cudaStream_t st);

struct AttnArgs {
    const void *q;
    void *out;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens;
    const int32_t *query_start_lens;
    int num_seqs;
    int num_tokens;
    int n_q_heads;
    float scale;
    void *workspace;
    size_t workspace_bytes;
    // the query rows' own K/V rows ([num_tokens, n_kv_heads, head_dim], pool dtype),
    // stored at their positions before they are read; nullptr: no append
    const void *k_new = nullptr, *v_new = nullptr;
};

// The query rows' K/V of an attention call (a.k_new, a.v_new) stored at their
// positions (slot from the block table), one warp per token.
int launch_kv_append_at_positions(const pk_pool *p, const AttnArgs &a, cudaStream_t st);

int launch_attention_generic(const pk_pool *p, const AttnArgs &a, cudaStream_t st);

// Tensor-core path: workspace sizing and launch.
size_t tc_workspace_bytes(const pk_pool *p, int num_seqs, int num_tokens, int n_q_heads,
                          int max_blocks_per_seq);
// Bytes at the start of every workspace that must be zero when a call starts
// (scheduler headers and split-K arrival counters); the same for every pool.
size_t tc_workspace_zeroed_bytes();
int tc_prepare_pool(pk_pool *p);  // occupancy queries, once per pool
int launch_attention_tc(const pk_pool *p, const AttnArgs &a, cudaStream_t st);

// The decode kernel's share of the workspace.
struct DecodeWs {
    void *header;
    int *counters;
    int *merge_plan;  // the block-streaming kernel's plan, for its merge kernel
    float *partial_o, *partial_lse;
    int cap_rows;
};
int decode_prepare_pool(pk_pool *p);
int decode_items_per_cta();
int launch_decode(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, cudaStream_t st);
// Block-streaming decode kernel: the one-query-token sequences of a batch, for
// groups of at most 8 q heads per kv head.  skip_chunks: the batch also holds
// sequences of several query tokens, which the chunk kernel serves (without
// it such a sequence is recorded as PK_ERR_BAD_INDEX).
int decode_blocks_prepare_pool(pk_pool *p);
int decode_blocks_chunks_per_cta();
bool decode_blocks_applies(const pk_pool *p, const AttnArgs &a);
int launch_decode_blocks(const pk_pool *p, const AttnArgs &a, const DecodeWs &w, bool skip_chunks,
                         bool behind_chunk, cudaStream_t st);
// 2-D TMA view of a pool (rows of head_dim bf16) with boxes of 64 columns x box_rows.
int encode_pool_map(CUtensorMap *map, void *base, const pk_pool *p, int box_rows);
// 3-D TMA view (column in panel, row, 64-column panel) with boxes of all panels x box_rows.
int encode_pool_map3(CUtensorMap *map, void *base, const pk_pool *p, int box_rows);
int chunk_prepare_pool(pk_pool *p);
// tcgen05 chunk kernel (head_dim 128, block_size a multiple of 16, g dividing 128).
// all_multi: serve every sequence of two or more query tokens (the one-token
// ones go to the block-streaming decode kernel); otherwise every sequence whose
// rows (query tokens x group heads) exceed one 16-row tile.
int chunk_umma_prepare_pool(pk_pool *p);
bool chunk_umma_applies(const pk_pool *p, const AttnArgs &a);
int launch_chunk_umma(const pk_pool *p, const AttnArgs &a, bool all_multi, cudaStream_t st);
// head dim 256: one 128-row tile per item, two S buffers in tensor memory
int chunk_umma256_prepare(pk_pool *p);
int launch_chunk_umma256(const pk_pool *p, const AttnArgs &a, bool all_multi, cudaStream_t st);
int launch_chunk(const pk_pool *p, const AttnArgs &a, void *header, cudaStream_t st);

}  // namespace pk
