// pk_paged_attention_noalloc: paged attention for callers that cannot
// allocate device memory.
//
// pk_paged_attention takes its scratch (the work-claim counter, the split-K
// arrival counters and the split-K partial results) from a caller-provided
// workspace.  Some callers cannot provide
// one: a plain C host program with no caching allocator, or a serving loop
// that reserves all free HBM for the KV pool up front, where a cudaMalloc on
// the request path would fail or stall the whole device.  This entry point
// takes its scratch from a fixed array in the library's own device memory
// instead, and allocates nothing.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes
// (32 MiB).  Every GPU that loads the library holds it until the process
// exits.  In host code the array's name is only a host-side stand-in, not a
// device address: passing it to a kernel would fault or, where the GPU can
// reach host memory, silently use the wrong memory.  The first call on each
// device therefore looks the real address up with cudaGetSymbolAddress, with
// that device current, and caches it; make that first call before any stream
// capture.
//
// All calls share the array and it keeps the last call's contents.  The only
// state a call relies on at its start is the work-claim counters and the
// split-K arrival counters, which must be zero; they sit in a region at the
// start of the array whose offsets and size are the same for every pool.  A
// completed call leaves them zeroed, but a call that gave up on a bounded wait
// (PK_ERR_TIMEOUT) may not, and nobody else can reach the array to clear it:
// so every call first zeroes that region on its own stream with
// cudaMemsetAsync (a few hundred KiB; it allocates nothing).  Everything else
// is written before it is read.  Two calls whose work overlaps on the GPU (on
// two streams, or from two host threads) race on the array and corrupt each
// other's results.  Serialise them.
#include <mutex>

#include "pk_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)PK_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_attention_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return pk::cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return pk::fail(PK_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attention_scratch);
        if (e != cudaSuccess) return pk::cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PK_OK;
}

}  // namespace

extern "C" int pk_paged_attention_noalloc(const pk_pool *pool, const void *q, void *out,
                                          const int32_t *block_tables, int max_blocks_per_seq,
                                          const int32_t *context_lens,
                                          const int32_t *query_start_lens, int num_seqs,
                                          int num_tokens, int n_q_heads, float scale,
                                          pk_stream_t stream) {
    if (!pool) return pk::fail(PK_ERR_INVALID_ARG, "pool is NULL");
    size_t need = 0;
    int rc = pk_attention_workspace_size(pool, num_seqs, num_tokens, n_q_heads,
                                         max_blocks_per_seq, &need);
    if (rc != PK_OK) return rc;
    if (need > kNoAllocScratchBytes)
        return pk::fail(PK_ERR_WORKSPACE,
                        "batch needs %zu bytes of scratch; the no-allocation entry point has "
                        "%zu (use pk_paged_attention with a workspace)",
                        need, kNoAllocScratchBytes);
    if (num_seqs == 0)  // argument checks only; nothing is queued
        return pk_paged_attention(pool, q, out, block_tables, max_blocks_per_seq, context_lens,
                                  query_start_lens, num_seqs, num_tokens, n_q_heads, scale, nullptr,
                                  0, stream);
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != pool->device)
        return pk::fail(PK_ERR_INVALID_ARG, "the pool's device must be current");
    void *scratch = nullptr;
    rc = scratch_on_current_device(&scratch);
    if (rc != PK_OK) return rc;
    if (pool->tc_path) {
        const cudaError_t e =
            cudaMemsetAsync(scratch, 0, pk::tc_workspace_zeroed_bytes(), (cudaStream_t)stream);
        if (e != cudaSuccess) return pk::cuda_fail(e, "clearing the scratch counters");
    }
    return pk_paged_attention(pool, q, out, block_tables, max_blocks_per_seq, context_lens,
                              query_start_lens, num_seqs, num_tokens, n_q_heads, scale, scratch,
                              kNoAllocScratchBytes, stream);
}
