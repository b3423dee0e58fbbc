/*
 * paged_kv.h -- C ABI of the paged KV cache library for NVIDIA B200 (sm_100a).
 *
 * The library implements the data path of PagedAttention with continuous
 * batching: a pool of fixed-size physical KV blocks, per-sequence block
 * tables, the attention kernel that gathers K/V through those tables
 * (decode rows and causal chunked-prefill rows, GQA), the slot-mapped append
 * of new tokens' K/V, the whole-block copy used by copy-on-write, and the
 * host-side block manager that produces tables, slots and copy pairs.
 *
 * Sources for what each call computes:
 *   [SN]  "PagedAttention & Continuous Batching" (study notes), sections
 *         "Block tables", "Copy-on-write", "Continuous batching", "Flow".
 *   [BP]  "Batching and PagedAttention", sections "Continuous batching",
 *         "PagedAttention", "Sharing blocks", "When blocks run out",
 *         "Choosing the block size".
 *   [DD]  "7.8 PagedAttention & continuous batching" (LLM deep dive),
 *         "01 Concept".
 *
 * Conventions (every call):
 *   - Returns int status: PK_OK (0) or one of the PK_ERR_* codes below.  On
 *     error nothing is launched and pk_last_error() describes the cause.
 *   - Device pointers belong to the caller and must stay valid until the work
 *     queued on `stream` has finished.  Calls are asynchronous on `stream`
 *     (a cudaStream_t; NULL is the legacy default stream).  Nothing
 *     synchronises except pk_check_device_errors.
 *   - Integer metadata that lives on the device (tables, lengths, slots,
 *     copy pairs) cannot be checked before launch.  Kernels check every
 *     block id and slot they dereference; a bad one is skipped (or replaced
 *     by block 0 in attention), never dereferenced, and
 *     PK_ERR_BAD_INDEX is recorded in the pool's device error word, which
 *     pk_check_device_errors reads.  Results of such a call are undefined.
 *   - Bounded waits: a pipeline wait that exceeds its iteration limit records
 *     PK_ERR_TIMEOUT in the same word and the kernel returns.
 *   - Stream order holds as for plain launches.  The kernels are launched as
 *     programmatic dependents of the kernel before them on `stream`, so a
 *     call's kernels may start while that kernel drains.  They wait for it
 *     (griddepcontrol.wait) before they touch the pool, the output or any
 *     scratch. Before that wait the attention kernels read only their plan
 *     inputs: q, the block tables, the context lengths and the query offsets.
 *     One obligation on the caller follows. A kernel of its own that
 *     immediately precedes an attention call on `stream` and signals its
 *     dependents early (griddepcontrol.launch_dependents) must not write
 *     those four arrays after the signal. Kernels that never signal, copies
 *     and events are unaffected.
 *   - Threading: calls on different pools may run concurrently; calls on
 *     one pk_bm must be serialised by the caller.
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pk_stream_t; /* same type as cudaStream_t */

enum {
    PK_OK = 0,
    PK_ERR_INVALID_ARG = 1,  /* bad host-side argument (shape, pointer, alignment) */
    PK_ERR_OOM = 2,          /* block manager: not enough free blocks; state unchanged */
    PK_ERR_UNSUPPORTED = 3,  /* dtype / geometry this build does not handle */
    PK_ERR_CUDA = 4,         /* a CUDA runtime call failed (message in pk_last_error) */
    PK_ERR_BAD_INDEX = 5,    /* device: a block id or slot outside the pool was skipped */
    PK_ERR_WORKSPACE = 6,    /* workspace smaller than pk_attention_workspace_size */
    PK_ERR_TIMEOUT = 7       /* device: a bounded pipeline wait ran out */
};

enum { PK_F32 = 0, PK_BF16 = 1 };

/* Thread-local description of the last error of this thread ("" if none). */
const char *pk_last_error(void);

/* Library version string. */
const char *pk_version(void);

/* ------------------------------------------------------------------------
 * KV pool  [SN "Block tables"; BP "PagedAttention" item 1; DD]
 *
 * GPU memory for one layer's cache is divided into num_blocks equal physical
 * blocks, each holding K and V of block_size tokens.  Layout (both pools):
 *     [num_blocks][n_kv_heads][block_size][head_dim]   row-major, dtype
 * so the K (or V) rows of one (block, kv head) are one contiguous chunk of
 * block_size * head_dim elements.  Token slot s (0 <= s < num_blocks *
 * block_size) is block s / block_size, offset s % block_size.
 *
 * k_base / v_base: device memory of that size, owned by the caller (e.g.
 * torch tensors), 16-byte aligned.  The library owns only the descriptor and
 * a 4-byte device error word, both released by pk_pool_destroy.
 * dtype: PK_F32 or PK_BF16.  head_dim: 1..256 (fast tensor-core path: bf16,
 * head_dim 64/128/256, block_size a multiple of 8, n_kv_heads <= 64; anything
 * else runs a general CUDA kernel).  The current CUDA device at create time is
 * the pool's device; later calls must be made with that device current.
 * ------------------------------------------------------------------------ */
typedef struct pk_pool pk_pool;

int pk_pool_create(int num_blocks, int block_size, int n_kv_heads, int head_dim, int dtype,
                   void *k_base, void *v_base, pk_pool **out);
int pk_pool_destroy(pk_pool *pool);

/* Which attention kernels serve this pool, fixed when it was created: a bit
 * set of the PK_PATH_* values below (0: the general kernel serves every call).
 *   PK_PATH_TENSOR_CORE    TMA loads and tensor-core attention (bf16 geometries
 *                          named above)
 *   PK_PATH_DECODE_BLOCKS  one-token rows stream whole blocks, all kv heads of a
 *                          group per TMA box (block-streaming decode kernel)
 *   PK_PATH_CHUNK_TCGEN05  prefill chunks run on tcgen05 with accumulators in
 *                          tensor memory (head_dim 64, 128 or 256, block_size a
 *                          multiple of 16); without it they run on mma.sync.  The library
 *                          leaves it off when the kernel was not compiled with
 *                          the register count its warp roles are laid out for,
 *                          or when PK_CHUNK_MMA_SYNC=1 is set in the environment.
 * Host only; nothing is launched. */
enum { PK_PATH_TENSOR_CORE = 1, PK_PATH_DECODE_BLOCKS = 2, PK_PATH_CHUNK_TCGEN05 = 4 };
int pk_pool_paths(const pk_pool *pool, int *paths_out);

/* Reads and clears the pool's device error word (synchronises `stream`).
 * *code_out = PK_OK or the first PK_ERR_BAD_INDEX / PK_ERR_TIMEOUT recorded. */
int pk_check_device_errors(const pk_pool *pool, pk_stream_t stream, int *code_out);

/* ------------------------------------------------------------------------
 * KV append  [SN "Flow" step 4 "Append KV into mapped blocks"; BP
 * "PagedAttention" item 3: blocks are filled on demand as tokens arrive]
 *
 * For every token t < num_tokens with slot = slot_mapping[t] >= 0:
 *     Kpool[slot / bs][h][slot % bs][:] = k[t][h][:]   for every kv head h
 *     Vpool[...] likewise from v.
 * k, v: device [num_tokens][n_kv_heads][head_dim] of the pool's dtype,
 * contiguous.  slot_mapping: device int64 [num_tokens]; a negative slot
 * skips the token; slots must be distinct within one call (otherwise which
 * token wins is undefined).  Bit-exact copy.
 * ------------------------------------------------------------------------ */
int pk_paged_kv_append(const pk_pool *pool, const void *k, const void *v,
                       const int64_t *slot_mapping, int num_tokens, pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Block copy (copy-on-write)  [SN "Copy-on-write": a write into a shared
 * block allocates a fresh block, copies, then writes; DD]
 *
 * For each pair i < n_pairs: block dst = src_dst_pairs[2i+1] receives a copy
 * of block src = src_dst_pairs[2i] -- all heads, all slots, K and V.
 * src_dst_pairs: device int32 [n_pairs][2].  Destinations must be distinct
 * and no destination may be a source in the same call (the pairs the block
 * manager emits satisfy both).  Bit-exact copy.
 * ------------------------------------------------------------------------ */
int pk_block_copy(const pk_pool *pool, const int32_t *src_dst_pairs, int n_pairs,
                  pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Block swap between the device pool and a host pool  [BP "When blocks run
 * out": a preempted request's blocks are swapped out to CPU memory and later
 * back, all blocks of a sequence together]
 *
 * host_k, host_v: page-locked host memory of num_host_blocks blocks with the
 * pool's block geometry and dtype ([H][n_kv_heads][block_size][head_dim]),
 * mapped for device access (cudaHostAlloc, or pinned torch tensors); the
 * call checks this with cudaPointerGetAttributes and returns
 * PK_ERR_INVALID_ARG otherwise.  pairs: device int32 [n_pairs][2]; to_host
 * != 0: (device block, host block), host block := device block; to_host == 0:
 * (host block, device block), device block := host block.  Whole blocks, K and
 * V, bit-exact; the destinations of one call must be distinct.  Ids outside
 * either pool are recorded as PK_ERR_BAD_INDEX and skipped.  Asynchronous on
 * the stream: the host pool must stay allocated, and its swapped-out blocks
 * must not be read on the host, until the stream has passed the call.
 * ------------------------------------------------------------------------ */
int pk_swap_blocks(const pk_pool *pool, void *host_k, void *host_v, int num_host_blocks,
                   const int32_t *pairs, int n_pairs, int to_host, pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Paged attention  [SN "Block tables": the kernel gathers through the table;
 * BP "PagedAttention" item 4; BP "Continuous batching": one step mixes
 * prefill chunks and decodes, long prompts are split into chunks]
 *
 * Batch of num_seqs sequences.  Sequence b has context_lens[b] = c_b tokens
 * stored in the pool (this step's new tokens included: append first, then
 * attend) and q_b = query_start_lens[b+1] - query_start_lens[b] >= 1 query
 * tokens, the last q_b of its context (q_b = 1: decode; q_b > 1: a chunk).
 * For query token i of b (logical position p = c_b - q_b + i) and q head h:
 *     kvh = h / (n_q_heads / n_kv_heads)
 *     K_j = Kpool[block_tables[b][j / bs]][kvh][j % bs][:]   (j = 0..p)
 *     out[t][h][:] = sum_j softmax_j(scale * q[t][h] . K_j) * V_j
 * computed with fp32 accumulation and an online softmax.
 *
 * q, out: device [num_tokens][n_q_heads][head_dim], the pool's dtype,
 *   contiguous; num_tokens = query_start_lens[num_seqs].
 * block_tables: device int32 [num_seqs][max_blocks_per_seq]; entries past
 *   ceil(c_b / bs) are never read.  context_lens: device int32 [num_seqs],
 *   1 <= c_b <= max_blocks_per_seq * bs.  query_start_lens: device int32
 *   [num_seqs + 1], query_start_lens[0] = 0, 1 <= q_b <= c_b.
 * n_q_heads % n_kv_heads == 0.
 * workspace: device scratch of at least pk_attention_workspace_size bytes,
 *   256-byte aligned, owned by the caller, not shared by calls in flight at
 *   the same time (two streams need two workspaces); it holds the work-claim
 *   counters, the split-K arrival counters and the split-K partial results.
 *   It must be zero-filled before its first use; every call that completes
 *   leaves the counters zeroed again, at offsets that are the same for every
 *   pool and batch, so a workspace can be reused across calls, batches and
 *   pools.  After a call that recorded PK_ERR_TIMEOUT, zero it again.
 * ------------------------------------------------------------------------ */
int pk_attention_workspace_size(const pk_pool *pool, int num_seqs, int num_tokens,
                                int n_q_heads, int max_blocks_per_seq, size_t *bytes_out);

int pk_paged_attention(const pk_pool *pool, const void *q, void *out,
                       const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, const int32_t *query_start_lens,
                       int num_seqs, int num_tokens, int n_q_heads, float scale,
                       void *workspace, size_t workspace_bytes, pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Append, then attend, in one call ([SN] "Flow": the step's new K/V go into
 * the blocks their table maps them to; [BP] "PagedAttention" item 4).
 *
 * The same as pk_paged_kv_append of the query rows' own K/V, followed by
 * pk_paged_attention with the same arguments. Query row t = query_start_lens[b]
 * + i of sequence b holds the K/V rows k[t], v[t] ([num_tokens][n_kv_heads]
 * [head_dim], the pool's dtype, contiguous, 16-byte aligned). They are stored
 * at position c_b - q_b + i, in block block_tables[b][pos / bs] at offset
 * pos % bs, before any attention reads them.
 *
 * The slots follow from the tables, so no slot_mapping is taken.
 *   - A decode-only batch on the block-streaming path (bf16, groups of at
 *     most 8): the decode kernel stores each row's K/V just before it loads
 *     the block holding it. No append kernel runs.
 *   - Otherwise (batches with prefill chunks, other geometries): an append
 *     kernel stores every row first, then attention runs.
 * Results, and the pool afterwards, equal those of the two separate calls.
 * A table entry outside the pool is recorded (PK_ERR_BAD_INDEX) and its row
 * is not stored. Errors: as pk_paged_attention, and PK_ERR_INVALID_ARG for
 * k or v NULL or misaligned when num_seqs > 0. With num_seqs == 0 the call
 * queues no work and may be given NULL arrays, as pk_paged_attention may.
 * ------------------------------------------------------------------------ */
int pk_paged_attention_append(const pk_pool *pool, const void *q, const void *k, const void *v,
                              void *out, const int32_t *block_tables, int max_blocks_per_seq,
                              const int32_t *context_lens, const int32_t *query_start_lens,
                              int num_seqs, int num_tokens, int n_q_heads, float scale,
                              void *workspace, size_t workspace_bytes, pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Paged attention without a caller workspace.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate
 * device memory, such as a C host program with no caching allocator, or a
 * serving loop that has reserved all free HBM for the KV pool, where a
 * cudaMalloc on the request path would fail or stall the device.
 *
 * Same arguments and results as pk_paged_attention, minus the workspace: the
 * scratch comes from a fixed array of PK_NOALLOC_SCRATCH_BYTES in the
 * library's own device memory, which every GPU that loads the library holds
 * until the process exits.  The call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine).  A batch whose scratch need
 * (pk_attention_workspace_size) exceeds the array is refused with
 * PK_ERR_WORKSPACE before anything is launched.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  All calls
 * share the array and it keeps the last call's contents; each call starts by
 * clearing the array's counter region on `stream` (cudaMemsetAsync, which
 * allocates nothing), so a call that recorded PK_ERR_TIMEOUT leaves nothing
 * stale for the next one.  Calls whose work overlaps on the GPU (two streams,
 * two host threads) race on the array and corrupt each other's results, so
 * serialise them.  num_seqs == 0 returns PK_OK with nothing queued.
 * ------------------------------------------------------------------------ */
#define PK_NOALLOC_SCRATCH_BYTES (32u << 20)

int pk_paged_attention_noalloc(const pk_pool *pool, const void *q, void *out,
                               const int32_t *block_tables, int max_blocks_per_seq,
                               const int32_t *context_lens, const int32_t *query_start_lens,
                               int num_seqs, int num_tokens, int n_q_heads, float scale,
                               pk_stream_t stream);

/* ------------------------------------------------------------------------
 * Host block manager  [SN "Block tables", "Copy-on-write"; BP
 * "PagedAttention", "Sharing blocks", "When blocks run out"; DD]
 *
 * Free list, per-sequence block tables, reference counts, fork and
 * copy-on-write, on the host.  Policy (fixed so that two implementations
 * produce the same tables): the free list is first-in first-out starting as
 * 0..num_blocks-1; a freed block joins its tail; freeing a sequence releases
 * its blocks from the last logical block to the first; sequence ids count up
 * from 0 over add_seq and fork.
 * ------------------------------------------------------------------------ */
typedef struct pk_bm pk_bm;

typedef struct {
    int64_t num_blocks;
    int64_t free_blocks;
    int64_t used_blocks;
    int64_t alloc_failures;   /* append_slots calls refused with PK_ERR_OOM */
    int64_t tail_waste_slots; /* unwritten slots over all blocks in use, each block once */
    int64_t num_seqs;
    int64_t host_blocks;      /* host (swap) pool size, 0 until pk_bm_set_host_blocks */
    int64_t host_free_blocks;
    int64_t prefix_lookups;   /* keys offered to pk_bm_add_seq_cached */
    int64_t prefix_hits;      /* of which served by a cached block */
    int64_t cached_blocks;    /* blocks registered in the prefix cache now */
    int64_t state_slots;      /* per-sequence state pool size, 0 without one */
    int64_t state_free_slots;
} pk_bm_stats;

int pk_bm_create(int num_blocks, int block_size, pk_bm **out);
int pk_bm_destroy(pk_bm *bm);
/* New empty sequence; its id in *seq_out (PK_ERR_OOM: no free state slot,
 * with a state pool). */
int pk_bm_add_seq(pk_bm *bm, int64_t *seq_out);
/* Reserve slots for the next n tokens of seq.  slots_out[n] receives the slot
 * id of each token.  If the sequence's last block is partly filled and shared
 * (reference count > 1) a fresh block is taken first and the pair
 * (old, new) is written to pairs_out (int32 [pairs_cap][2]); *n_pairs_out is
 * the number of pairs (0 or 1).  The caller must run pk_block_copy on the
 * pairs before appending.  PK_ERR_OOM: not enough free blocks; nothing
 * changed. */
int pk_bm_append_slots(pk_bm *bm, int64_t seq, int n, int64_t *slots_out, int32_t *pairs_out,
                       int pairs_cap, int *n_pairs_out);
/* One token for each of seqs[0..n-1], in order, as append_slots(seq, 1) each:
 * slots_out[i] its slot, pairs_out (int32 [n][2]) the copy-on-write pairs in
 * order (*n_pairs_out of them).  Stops, without counting an allocation
 * failure, at the first sequence whose token needs a block when none is free:
 * *n_done_out sequences got their token.  An unknown or swapped-out sequence
 * ends the call with PK_ERR_INVALID_ARG; the ones before it keep their tokens
 * (*n_done_out, *n_pairs_out and their slots and pairs say which). */
int pk_bm_append_one_each(pk_bm *bm, const int64_t *seqs, int n, int64_t *slots_out, int32_t *pairs_out,
                          int *n_pairs_out, int *n_done_out);
/* Blocks append_slots(seq, n) would take from the free list. */
int pk_bm_blocks_needed(const pk_bm *bm, int64_t seq, int n, int *needed_out);
/* New sequence sharing all of parent's blocks (reference counts + 1). */
int pk_bm_fork(pk_bm *bm, int64_t parent, int64_t *child_out);
/* Drop seq; blocks no longer referenced return to the free list. */
int pk_bm_free(pk_bm *bm, int64_t seq);
/* Swapping [BP "When blocks run out": a preempted request's blocks are
 * swapped out to CPU memory, or freed and recomputed later; all blocks of a
 * sequence are evicted together].
 * pk_bm_set_host_blocks gives the manager a host pool of num_host_blocks
 * blocks (once; FIFO free list 0..H-1).
 * pk_bm_swap_out moves every block of a resident seq to the host pool:
 * pairs_out (int32 [pairs_cap][2]) receives one (device block, host block)
 * pair per table entry in logical order, the device blocks return to the free
 * list (last logical block first) and the table now names host blocks.  The
 * caller runs pk_swap_blocks(..., to_host = 1) on the pairs before anything
 * else writes those device blocks.  PK_ERR_UNSUPPORTED: the sequence shares a
 * block (reference count > 1); PK_ERR_OOM: too few free host blocks; nothing
 * changes in either case.
 * pk_bm_swap_in is the reverse: (host block, device block) pairs, run with
 * to_host = 0; PK_ERR_OOM: too few free device blocks, nothing changed.
 * A swapped sequence accepts only swap_in, free (its host blocks return),
 * block_table (host ids), seq_len and is_swapped; other calls return
 * PK_ERR_INVALID_ARG. */
int pk_bm_set_host_blocks(pk_bm *bm, int num_host_blocks);
int pk_bm_swap_out(pk_bm *bm, int64_t seq, int32_t *pairs_out, int pairs_cap, int *n_pairs_out);
int pk_bm_swap_in(pk_bm *bm, int64_t seq, int32_t *pairs_out, int pairs_cap, int *n_pairs_out);
int pk_bm_is_swapped(const pk_bm *bm, int64_t seq, int *swapped_out);
/* Prefix cache [BP "Sharing blocks": requests that share a system prompt can
 * share its blocks; DD: requests with an identical prompt prefix point at the
 * same read-only blocks, and the prefix hit rate is a metric to watch].
 * keys[i] is the caller's name for the token prefix 0 .. (i+1)*block_size - 1
 * (for example a chained hash of the token ids).
 * pk_bm_cache_blocks registers seq's first n_keys logical blocks, which must
 * be full (n_keys * block_size <= length; PK_ERR_INVALID_ARG otherwise), under
 * keys[]; a key already cached, or a block already registered, keeps its
 * entry.  pk_bm_add_seq_cached creates a sequence that starts on the cached
 * blocks of the longest cached prefix of keys[] (each count + 1; length
 * *n_hit_out * block_size); the caller then appends only the tokens after it.
 * pk_bm_cached_prefix reports that prefix length without changing anything.
 * An entry lives while its block is referenced: it leaves the cache when the
 * block returns to the free list.  Cached blocks are full, so appends never
 * write into them. */
int pk_bm_cache_blocks(pk_bm *bm, int64_t seq, const uint64_t *keys, int n_keys);
int pk_bm_cached_prefix(const pk_bm *bm, const uint64_t *keys, int n_keys, int *n_hit_out);
int pk_bm_add_seq_cached(pk_bm *bm, const uint64_t *keys, int n_keys, int64_t *seq_out, int *n_hit_out);
/* Two pools [DD: a hybrid model's attention layers keep growing, paged KV,
 * its other layers a fixed-size state per sequence; the server manages two
 * pools with different lifecycles].  pk_bm_set_state_slots (once, before any
 * sequence exists) adds a pool of num_slots state slots: every sequence takes
 * one when it is created (add_seq, add_seq_cached, fork) and returns it when
 * freed; with no free slot those calls return PK_ERR_OOM and change nothing.
 * A fork's slot is new: the caller copies the parent's state into it.  A
 * swapped-out sequence keeps its slot.  pk_bm_state_slot gives a sequence's
 * slot (-1 without a state pool). */
int pk_bm_set_state_slots(pk_bm *bm, int num_slots);
int pk_bm_state_slot(const pk_bm *bm, int64_t seq, int *slot_out);
/* Copy seq's block table (ceil(len / bs) ids) into out[cap]; *n_out = count. */
int pk_bm_block_table(const pk_bm *bm, int64_t seq, int32_t *out, int cap, int *n_out);
/* Fill out[n_seqs][width] (int32, row-major) with the tables of seqs[], -1 padded. */
int pk_bm_fill_tables(const pk_bm *bm, const int64_t *seqs, int n_seqs, int32_t *out, int width);
int pk_bm_seq_len(const pk_bm *bm, int64_t seq, int64_t *len_out);
int pk_bm_refcount(const pk_bm *bm, int32_t block, int *count_out);
int pk_bm_get_stats(const pk_bm *bm, pk_bm_stats *out);
/* Free device blocks now (stats' free_blocks, without the walk over every
 * block that the tail-waste count needs). */
int pk_bm_num_free(const pk_bm *bm, int *free_out);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
