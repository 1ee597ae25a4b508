/*
 * oracle.c -- plain, slow, fp64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file;
 * only the tests, the smoke check and the benchmark's CPU baseline do.  It
 * shares no code, header or constant with the CUDA library.
 *
 * What it computes (each function cites the passage it follows):
 *
 *   Paged attention looks up each cached key and value of a request through
 *   its block table, whatever pool position the block holds ("What vLLM Is
 *   and Why It Exists", section "The idea vLLM started from: pages"); keys
 *   and values that are consecutive in the sequence need not be consecutive
 *   in memory ("vLLM Solved the Wrong Bottleneck...", section "Paged
 *   Attention").  Paging only
 *   changes where the bytes live, so the result is ordinary softmax
 *   attention of one query token over the n cached tokens, written here as
 *   its definition:
 *
 *       x_i   = scale * sum_d q[d] * K_i[d]            (i = 0..n-1)
 *       w_i   = exp(x_i - max_j x_j)
 *       out   = sum_i w_i * V_i / sum_i w_i
 *
 *   where token i of sequence s lives in physical block
 *   block_tables[s][i / block_size] at offset i % block_size (day-9 post,
 *   section "Idea 1: PagedAttention": the block table takes a logical block
 *   number to a physical block of GPU memory).
 *
 * Readings where the pages are silent (listed with the rest of the design):
 *   - cache layout [num_blocks][num_kv_heads][block_size][head_dim];
 *   - query head h reads KV head h / (num_q_heads / num_kv_heads);
 *   - only tokens 0..n-1 are read; other slots may hold anything (NaN);
 *   - a context of length 0 gives an all-zero output;
 *   - a negative slot id in the slot write means "no token": skipped.
 *
 * Error bits returned (the documented device contract, retyped here):
 *   1 = a live block-table entry outside [0, num_blocks)   (row -> zeros)
 *   2 = a context length outside [0, min(max_context_len,
 *       max_blocks_per_seq * block_size)]                 (row -> zeros)
 *   4 = a slot id >= num_blocks * block_size               (token skipped)
 *   8 = a copy pair with an id outside [0, num_blocks) or src == dst (skipped)
 *  32 = query rows of a sequence out of order or more than its length (rows -> zeros)
 *
 * Element types: 0 = IEEE fp32, 1 = bf16 (the upper 16 bits of an fp32; its
 * widening to fp32 is exact).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double elem(const void *base, size_t i, int dtype)
{
    if (dtype == 0)
        return (double)((const float *)base)[i];
    uint32_t u = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Check sequence s: its length and every live table entry.  Returns the
 * error bits that make its output rows zero (0 when the row is computable). */
static int check_seq(const int32_t *table, int n, int num_blocks, int block_size,
                     int max_blocks_per_seq, int max_context_len)
{
    if (n < 0 || n > max_context_len || n > max_blocks_per_seq * block_size)
        return 2;
    int nb = (n + block_size - 1) / block_size;
    for (int j = 0; j < nb; ++j)
        if (table[j] < 0 || table[j] >= num_blocks)
            return 1;
    return 0;
}

/* Offset (in elements) of token i's head-g row in the cache. */
static size_t row_offset(const int32_t *table, int i, int g, int num_kv_heads,
                         int block_size, int head_dim)
{
    size_t b = (size_t)table[i / block_size];
    size_t off = (size_t)(i % block_size);
    return ((b * (size_t)num_kv_heads + (size_t)g) * (size_t)block_size + off) * (size_t)head_dim;
}

/*
 * out[s][h][d] (fp64) = attention of q[s][h] over the context_lens[s] cached
 * tokens of sequence s.  The definition, one (sequence, head) at a time.
 */
int oracle_paged_decode(double *out, const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens,
                        int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int max_blocks_per_seq, int num_blocks,
                        int max_context_len, double scale, int dtype)
{
    const int group = num_q_heads / num_kv_heads;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int s = 0; s < num_seqs; ++s) {
        for (int h = 0; h < num_q_heads; ++h) {
            double *o = out + ((size_t)s * num_q_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
            const int n = context_lens[s];
            int bad = check_seq(table, n, num_blocks, block_size, max_blocks_per_seq,
                                max_context_len);
            if (bad) {
                err |= bad;
                continue;
            }
            if (n == 0)
                continue;
            const int g = h / group;
            const size_t qoff = ((size_t)s * num_q_heads + h) * head_dim;
            double *x = (double *)malloc(sizeof(double) * (size_t)n);
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                double dot = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    dot += elem(q, qoff + d, dtype) * elem(k_cache, ro + d, dtype);
                x[i] = scale * dot;
                if (x[i] > m)
                    m = x[i];
            }
            double denom = 0.0;
            for (int i = 0; i < n; ++i) {
                double w = exp(x[i] - m);
                denom += w;
                size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                for (int d = 0; d < head_dim; ++d)
                    o[d] += w * elem(v_cache, ro + d, dtype);
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= denom;
            free(x);
        }
    }
    return err;
}

/*
 * Several query tokens per sequence (a chunk of a prompt, or tokens checked
 * together), each seeing the cache up to its own position.  The cache grows
 * by the chunk's tokens ("vLLM Solved the Wrong Bottleneck...", section
 * "Paged Attention") before they attend, and the chunk is the last
 * Q = query_start[s+1] - query_start[s] of the n = context_lens[s] cached
 * tokens, so query row j of sequence s (global row query_start[s] + j) sits
 * at position p = n - Q + j and attends to tokens 0..p only (causal):
 *
 *   out[r][h][:] = sum_{i<=p} exp(x_i - m) V_i / sum_{i<=p} exp(x_i - m),
 *   x_i = scale * q[r][h] . K_i,  m = max_{i<=p} x_i.
 *
 * A sequence whose query_start pair is out of order, or whose Q exceeds n,
 * gets zero rows and error bit 32; the checks of oracle_paged_decode apply
 * to n and the table as well.  q and out are [query_start[S]][Hq][D].
 */
int oracle_paged_prefill(double *out, const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *block_tables, const int32_t *context_lens,
                         const int32_t *query_start, int num_seqs, int num_query_tokens,
                         int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                         int max_blocks_per_seq, int num_blocks, int max_context_len,
                         double scale, int dtype)
{
    const int group = num_q_heads / num_kv_heads;
    int err = 0;
    for (size_t i = 0; i < (size_t)num_query_tokens * num_q_heads * head_dim; ++i)
        out[i] = 0.0;
#pragma omp parallel for schedule(dynamic) reduction(| : err)
    for (int s = 0; s < num_seqs; ++s) {
        const int r0 = query_start[s], r1 = query_start[s + 1];
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
        const int n = context_lens[s];
        if (r0 < 0 || r1 < r0 || r1 > num_query_tokens) {
            err |= 32;
            continue;
        }
        int bad = check_seq(table, n, num_blocks, block_size, max_blocks_per_seq,
                            max_context_len);
        if (!bad && r1 - r0 > n)
            bad = 32;
        if (bad) {
            err |= bad;
            continue;
        }
        const int Q = r1 - r0;
        double *x = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        for (int j = 0; j < Q; ++j) {
            const int p = n - Q + j;  /* position of this query token */
            for (int h = 0; h < num_q_heads; ++h) {
                const int g = h / group;
                const size_t qoff = ((size_t)(r0 + j) * num_q_heads + h) * head_dim;
                double *o = out + qoff;
                double m = -INFINITY;
                for (int i = 0; i <= p; ++i) {
                    size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += elem(q, qoff + d, dtype) * elem(k_cache, ro + d, dtype);
                    x[i] = scale * dot;
                    if (x[i] > m)
                        m = x[i];
                }
                double denom = 0.0;
                for (int i = 0; i <= p; ++i) {
                    double w = exp(x[i] - m);
                    denom += w;
                    size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                    for (int d = 0; d < head_dim; ++d)
                        o[d] += w * elem(v_cache, ro + d, dtype);
                }
                for (int d = 0; d < head_dim; ++d)
                    o[d] /= denom;
            }
        }
        free(x);
    }
    return err;
}

/*
 * The same attention computed in partitions of partition_size tokens
 * (tokens [j*P, min(n, (j+1)*P)) for j = 0, 1, ...), each partition keeping
 * its own max m_j, sum l_j = sum exp(x_i - m_j) and normalised output
 * o_j = sum exp(x_i - m_j) V_i / l_j, then merged by log-sum-exp:
 *
 *     M = max_j m_j,  c_j = l_j * exp(m_j - M),  out = sum_j c_j o_j / sum_j c_j.
 *
 * This is the split-K form a long context takes (partitions of 512 tokens
 * merged by log-sum-exp, as the long-context workload asks).  It must equal
 * oracle_paged_decode up to rounding; the tests pin that identity.
 */
int oracle_paged_decode_partitioned(double *out, const void *q, const void *k_cache,
                                    const void *v_cache, const int32_t *block_tables,
                                    const int32_t *context_lens, int num_seqs, int num_q_heads,
                                    int num_kv_heads, int head_dim, int block_size,
                                    int max_blocks_per_seq, int num_blocks, int max_context_len,
                                    double scale, int dtype, int partition_size)
{
    if (partition_size <= 0)
        return -1;
    const int group = num_q_heads / num_kv_heads;
    int err = 0;
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(| : err)
    for (int s = 0; s < num_seqs; ++s) {
        for (int h = 0; h < num_q_heads; ++h) {
            double *o = out + ((size_t)s * num_q_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
            const int n = context_lens[s];
            int bad = check_seq(table, n, num_blocks, block_size, max_blocks_per_seq,
                                max_context_len);
            if (bad) {
                err |= bad;
                continue;
            }
            if (n == 0)
                continue;
            const int g = h / group;
            const size_t qoff = ((size_t)s * num_q_heads + h) * head_dim;
            const int nparts = (n + partition_size - 1) / partition_size;
            double *pm = (double *)malloc(sizeof(double) * (size_t)nparts);
            double *pl = (double *)malloc(sizeof(double) * (size_t)nparts);
            double *po = (double *)calloc((size_t)nparts * (size_t)head_dim, sizeof(double));
            double *x = (double *)malloc(sizeof(double) * (size_t)partition_size);
            for (int j = 0; j < nparts; ++j) {
                const int lo = j * partition_size;
                const int hi = lo + partition_size < n ? lo + partition_size : n;
                double m = -INFINITY;
                for (int i = lo; i < hi; ++i) {
                    size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += elem(q, qoff + d, dtype) * elem(k_cache, ro + d, dtype);
                    x[i - lo] = scale * dot;
                    if (x[i - lo] > m)
                        m = x[i - lo];
                }
                double l = 0.0;
                double *oj = po + (size_t)j * head_dim;
                for (int i = lo; i < hi; ++i) {
                    double w = exp(x[i - lo] - m);
                    l += w;
                    size_t ro = row_offset(table, i, g, num_kv_heads, block_size, head_dim);
                    for (int d = 0; d < head_dim; ++d)
                        oj[d] += w * elem(v_cache, ro + d, dtype);
                }
                for (int d = 0; d < head_dim; ++d)
                    oj[d] /= l;
                pm[j] = m;
                pl[j] = l;
            }
            double M = -INFINITY;
            for (int j = 0; j < nparts; ++j)
                if (pm[j] > M)
                    M = pm[j];
            double csum = 0.0;
            for (int j = 0; j < nparts; ++j) {
                double c = pl[j] * exp(pm[j] - M);
                csum += c;
                for (int d = 0; d < head_dim; ++d)
                    o[d] += c * po[(size_t)j * head_dim + d];
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= csum;
            free(pm);
            free(pl);
            free(po);
            free(x);
        }
    }
    return err;
}

/*
 * Slot write: each step's new key/value of token t, for every KV head, goes
 * to the cache slot slot_mapping[t] = block * block_size + offset.  The cache
 * gets longer with every generated token ("vLLM Solved the Wrong
 * Bottleneck...", section "Paged Attention"), and every request gains one
 * token per step ("What vLLM Is and Why It Exists", section "A picture").  A pure byte
 * copy: key/value are [num_tokens][num_kv_heads][head_dim].
 */
int oracle_reshape_and_cache(void *k_cache, void *v_cache, const void *key, const void *value,
                             const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                             int head_dim, int block_size, int num_blocks, int elem_bytes)
{
    int err = 0;
    const size_t row = (size_t)head_dim * (size_t)elem_bytes;
    for (int t = 0; t < num_tokens; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size) {
            err |= 4;
            continue;
        }
        const size_t b = (size_t)(slot / block_size), off = (size_t)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t dst = ((b * (size_t)num_kv_heads + (size_t)h) * (size_t)block_size + off) * row;
            size_t src = ((size_t)t * (size_t)num_kv_heads + (size_t)h) * row;
            memcpy((char *)k_cache + dst, (const char *)key + src, row);
            memcpy((char *)v_cache + dst, (const char *)value + src, row);
        }
    }
    return err;
}

/*
 * Copy-on-write: a shared block is duplicated, alone, when one of its
 * sharers must change it (day-9 post, section "Idea 1: PagedAttention").  For each
 * pair (src, dst) of block_mapping ([num_pairs][2]) the whole physical block
 * src (all KV heads, all slots) is copied to dst, in K and in V.
 */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_mapping, int num_pairs,
                       int num_kv_heads, int head_dim, int block_size, int num_blocks,
                       int elem_bytes)
{
    int err = 0;
    const size_t blk = (size_t)num_kv_heads * (size_t)block_size * (size_t)head_dim *
                       (size_t)elem_bytes;
    for (int p = 0; p < num_pairs; ++p) {
        const int32_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || src == dst) {
            err |= 8;
            continue;
        }
        memcpy((char *)k_cache + (size_t)dst * blk, (const char *)k_cache + (size_t)src * blk, blk);
        memcpy((char *)v_cache + (size_t)dst * blk, (const char *)v_cache + (size_t)src * blk, blk);
    }
    return err;
}
