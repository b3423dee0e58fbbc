/*
 * Oracle (test infrastructure only): plain float64 CPU definition of paged
 * attention.  Only tests/, the package smoke check and the bench's
 * CPU-baseline leg may load this file's library.  It shares no code, header
 * or constant with the CUDA path.
 *
 * What is computed, and where it is stated:
 *
 *  - paged attention: the attention kernel gathers keys and values through
 *    the sequence's block table instead of reading one contiguous slab
 *    [PagedAttention & Continuous Batching (study notes), "Block tables";
 *    Batching and PagedAttention, "PagedAttention", item 4].  Paging changes
 *    only where a token's K/V sits, so the result is ordinary softmax
 *    attention over the sequence's logical tokens; this file writes that
 *    definition out.
 *  - chunked prefill [Batching and PagedAttention, "Continuous batching":
 *    long prompts are split into chunks run across several steps]: a chunk of
 *    q query tokens of a sequence whose context (the chunk included) has c
 *    tokens holds logical positions c-q .. c-1; each of them sees every key
 *    at a position <= its own.  A decode step is the chunk with q = 1.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - pool layout: K and V pools are each [num_blocks][n_kv_heads][block_size]
 *    [head_dim]; logical token j of a sequence lives in physical block
 *    table[j / block_size] at slot j % block_size.
 *  - GQA: q head h reads kv head h / (n_q_heads / n_kv_heads).
 *  - softmax uses the natural exponential of scale * (q . k), max-subtracted.
 *
 * Everything is float64 and follows the definition one query row at a time:
 * no tiling, no online softmax, no reordering of the sums.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_INDEX 2
#define ORACLE_NO_MEMORY 3

/* Storage types the oracle reads.  Every value is widened exactly to double
 * on load (a bfloat16 is the upper half of an IEEE binary32). */
#define ORACLE_F64 0
#define ORACLE_F32 1
#define ORACLE_BF16 2

static double load_elem(const void *base, int64_t idx, int elt) {
    if (elt == ORACLE_F64) return ((const double *)base)[idx];
    if (elt == ORACLE_F32) return (double)((const float *)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Flat index of element (block, head, slot, 0) of a pool laid out as
 * [num_blocks][n_kv_heads][block_size][head_dim]. */
static int64_t pool_row(int64_t block, int head, int slot, int n_kv_heads, int block_size,
                        int head_dim) {
    return ((block * n_kv_heads + head) * (int64_t)block_size + slot) * head_dim;
}

typedef struct {
    const void *q, *k_pool, *v_pool;
    int q_elt, kv_elt;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens, *query_start_lens;
    int num_seqs, num_tokens, n_q_heads, n_kv_heads, head_dim, block_size, num_blocks;
    double scale;
} batch_t;

/*
 * Checks the batch description; returns ORACLE_OK or an error code.
 * Requirements: 1 <= q_b <= c_b for every sequence, query_start_lens
 * increasing from 0 to num_tokens, every block id a row of the pool.
 */
int oracle_check_batch(const int32_t *block_tables, int max_blocks_per_seq,
                       const int32_t *context_lens, const int32_t *query_start_lens,
                       int num_seqs, int num_tokens, int block_size, int num_blocks) {
    if (num_seqs < 0 || block_size < 1 || max_blocks_per_seq < 0 || num_tokens < 0)
        return ORACLE_BAD_ARG;
    if (query_start_lens[0] != 0 || query_start_lens[num_seqs] != num_tokens) return ORACLE_BAD_ARG;
    for (int b = 0; b < num_seqs; ++b) {
        int q = query_start_lens[b + 1] - query_start_lens[b];
        int c = context_lens[b];
        if (q < 1 || c < q) return ORACLE_BAD_ARG;
        int nblk = (c + block_size - 1) / block_size;
        if (nblk > max_blocks_per_seq) return ORACLE_BAD_ARG;
        for (int j = 0; j < nblk; ++j) {
            int32_t id = block_tables[(int64_t)b * max_blocks_per_seq + j];
            if (id < 0 || id >= num_blocks) return ORACLE_BAD_INDEX;
        }
    }
    return ORACLE_OK;
}

/*
 * One output row, for query token t (of sequence b) and q head h:
 *
 *   p    = c_b - q_b + (t - qsl_b)       logical position of the query token
 *   kvh  = h / (n_q_heads / n_kv_heads)
 *   K_j  = Kpool[table_b[j / bs]][kvh][j % bs][:]   for j = 0..p  (V_j alike)
 *   s_j  = scale * sum_e q[e] * K_j[e]
 *   w_j  = exp(s_j - max_j s_j)
 *   out  = sum_j w_j V_j / sum_j w_j
 *
 * w is scratch of at least p + 1 doubles.
 */
static void attend_row(const batch_t *a, int b, int t, int h, double *w, double *orow) {
    const int c = a->context_lens[b];
    const int qlen = a->query_start_lens[b + 1] - a->query_start_lens[b];
    const int pos = c - qlen + (t - a->query_start_lens[b]);
    const int kvh = h / (a->n_q_heads / a->n_kv_heads);
    const int bs = a->block_size, d = a->head_dim;
    const int32_t *table = a->block_tables + (int64_t)b * a->max_blocks_per_seq;
    const int64_t qoff = ((int64_t)t * a->n_q_heads + h) * d;

    double smax = -INFINITY;
    for (int j = 0; j <= pos; ++j) {
        const int64_t koff = pool_row(table[j / bs], kvh, j % bs, a->n_kv_heads, bs, d);
        double s = 0.0;
        for (int e = 0; e < d; ++e)
            s += load_elem(a->q, qoff + e, a->q_elt) * load_elem(a->k_pool, koff + e, a->kv_elt);
        w[j] = a->scale * s;
        if (w[j] > smax) smax = w[j];
    }
    double denom = 0.0;
    for (int j = 0; j <= pos; ++j) {
        w[j] = exp(w[j] - smax);
        denom += w[j];
    }
    for (int e = 0; e < d; ++e) orow[e] = 0.0;
    for (int j = 0; j <= pos; ++j) {
        const int64_t voff = pool_row(table[j / bs], kvh, j % bs, a->n_kv_heads, bs, d);
        for (int e = 0; e < d; ++e) orow[e] += w[j] * load_elem(a->v_pool, voff + e, a->kv_elt);
    }
    for (int e = 0; e < d; ++e) orow[e] /= denom;
}

static int seq_of_token(const batch_t *a, int t) {
    int lo = 0, hi = a->num_seqs - 1; /* last b with qsl[b] <= t */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (a->query_start_lens[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

static int max_context(const batch_t *a) {
    int m = 1;
    for (int b = 0; b < a->num_seqs; ++b)
        if (a->context_lens[b] > m) m = a->context_lens[b];
    return m;
}

/*
 * Evaluates attend_row for n_rows (token, head) pairs; rows == NULL means all
 * num_tokens * n_q_heads rows in order (token-major), otherwise rows holds
 * n_rows pairs (token, head).  out is [n_rows][head_dim] float64.
 * Rows are independent, so OpenMP spreads them over the host cores.
 */
static int run_rows(const batch_t *a, const int32_t *rows, int64_t n_rows, double *out) {
    if (a->n_q_heads < 1 || a->n_kv_heads < 1 || a->n_q_heads % a->n_kv_heads != 0 ||
        a->head_dim < 1 || a->q_elt < 0 || a->q_elt > 2 || a->kv_elt < 0 || a->kv_elt > 2)
        return ORACLE_BAD_ARG;
    int rc = oracle_check_batch(a->block_tables, a->max_blocks_per_seq, a->context_lens,
                                a->query_start_lens, a->num_seqs, a->num_tokens, a->block_size,
                                a->num_blocks);
    if (rc != ORACLE_OK) return rc;
    if (rows)
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[2 * r] < 0 || rows[2 * r] >= a->num_tokens || rows[2 * r + 1] < 0 ||
                rows[2 * r + 1] >= a->n_q_heads)
                return ORACLE_BAD_ARG;
    const int wlen = max_context(a);
    int failed = 0;
#pragma omp parallel
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)wlen);
        if (!w) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (!w) continue;
            int t = rows ? rows[2 * r] : (int)(r / a->n_q_heads);
            int h = rows ? rows[2 * r + 1] : (int)(r % a->n_q_heads);
            attend_row(a, seq_of_token(a, t), t, h, w, out + r * a->head_dim);
        }
        free(w);
    }
    return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/*
 * Full batch: out[t][h][:] for every query token t and q head h.
 * q is [num_tokens][n_q_heads][head_dim] of q_elt; the pools are
 * [num_blocks][n_kv_heads][block_size][head_dim] of kv_elt; out is float64.
 */
int oracle_paged_attention(const void *q, int q_elt, const void *k_pool, const void *v_pool,
                           int kv_elt, const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, const int32_t *query_start_lens,
                           int num_seqs, int num_tokens, int n_q_heads, int n_kv_heads,
                           int head_dim, int block_size, int num_blocks, double scale,
                           double *out) {
    batch_t a = {q, k_pool, v_pool, q_elt, kv_elt, block_tables, max_blocks_per_seq,
                 context_lens, query_start_lens, num_seqs, num_tokens, n_q_heads,
                 n_kv_heads, head_dim, block_size, num_blocks, scale};
    return run_rows(&a, NULL, (int64_t)num_tokens * n_q_heads, out);
}

/*
 * Sampled rows: the same definition for the listed (token, q head) pairs
 * only (rows is [n_rows][2]); out is [n_rows][head_dim].  Used where the
 * whole batch is too large for a float64 CPU pass.
 */
int oracle_paged_attention_rows(const void *q, int q_elt, const void *k_pool,
                                const void *v_pool, int kv_elt, const int32_t *block_tables,
                                int max_blocks_per_seq, const int32_t *context_lens,
                                const int32_t *query_start_lens, int num_seqs, int num_tokens,
                                int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                                int num_blocks, double scale, const int32_t *rows,
                                int64_t n_rows, double *out) {
    batch_t a = {q, k_pool, v_pool, q_elt, kv_elt, block_tables, max_blocks_per_seq,
                 context_lens, query_start_lens, num_seqs, num_tokens, n_q_heads,
                 n_kv_heads, head_dim, block_size, num_blocks, scale};
    return run_rows(&a, rows, n_rows, out);
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
