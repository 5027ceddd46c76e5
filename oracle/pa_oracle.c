/*
 * pa_oracle.c -- plain CPU oracle for paged KV-cache decode attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg and reference arm call this file. The CUDA library never links,
 * loads or calls it, and it shares no code, header or table with that library.
 *
 * Everything here is single-threaded, in double precision, and written in the
 * order the pages describe the method, with no blocking, fusion or reordering.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "PagedAttention 源码解析：KV Cache 怎么管理" (coreui.cn)
 *   [P2] "PagedAttention原理与KV Cache显存优化" (xdnf.cn)
 *   [P3] "Ascend C算子开发高阶实战：实现高性能KV Cache管理与PagedAttention融合算子" (cann.csdn.net)
 *   [P4] "PagedAttention 实现细节" (pyllm.pages.dev, vLLM series)
 *   [P5] "Ascend平台下的PageAttention优化实践" (jsqmd.com)
 *
 * Layouts (fixed for the whole project):
 *   query / out      [num_seqs, num_heads, head_dim]
 *   k_cache/v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
 *                    (the kernel view of [P4] §3.1, separate K and V pools)
 *   block_tables     [num_seqs, max_blocks_per_seq] int32
 *   context_lens     [num_seqs] int32
 *   slot_mapping     [num_tokens] int32, slot = block * block_size + offset
 *
 * Return codes: 0 = ok, negative = the inputs break a stated precondition
 * (the code says which); nothing is written past the point of failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_BAD_ARG -1
#define OR_TABLE_TOO_SHORT -2
#define OR_BAD_BLOCK_ID -3
#define OR_BAD_SLOT -4
#define OR_NO_MEMORY -5

/* Number of blocks a sequence of n tokens occupies: ceil(n / block_size).
 * [P3] §1.2 (45 tokens -> 3 blocks, 100 -> 7 at block size 16);
 * [P2] §3.2 (17 tokens -> 2 blocks); [P4] §3.1 demo (50 tokens -> 4 blocks). */
int oracle_blocks_needed(int num_tokens, int block_size)
{
    if (num_tokens < 0 || block_size <= 0)
        return OR_BAD_ARG;
    return (num_tokens + block_size - 1) / block_size;
}

/* Offset, in elements, of row (block, kv_head, offset) of a
 * [num_blocks, num_kv_heads, block_size, head_dim] pool. */
static size_t pool_row(int block, int kv_head, int offset, int num_kv_heads,
                       int block_size, int head_dim)
{
    return (((size_t)block * num_kv_heads + kv_head) * block_size + offset) *
           (size_t)head_dim;
}

/* Checks that sequence s's first ceil(L / block_size) table entries are valid
 * physical ids. Entries beyond that are never read ([P4] §3.1: the gather
 * stops once the valid tokens are collected). */
static int check_table_row(const int32_t *row, int L, int block_size,
                           int max_blocks_per_seq, int num_blocks)
{
    int nb = oracle_blocks_needed(L, block_size);
    if (nb < 0)
        return OR_BAD_ARG;
    if (nb > max_blocks_per_seq)
        return OR_TABLE_TOO_SHORT;
    for (int j = 0; j < nb; ++j)
        if (row[j] < 0 || row[j] >= num_blocks)
            return OR_BAD_BLOCK_ID;
    return OR_OK;
}

/* Gathers the first L tokens of sequence s (kv head kvh) into contiguous
 * K[L, D] and V[L, D]: token t lives in physical block
 * block_table[t / block_size] at offset t % block_size.
 * [P2] §3.1 (logical block t // 16, offset t % 16); [P4] §3.1
 * gather_kv_from_blocks (walk the table, trim the last block). */
static void gather_tokens(double *K, double *V, const double *k_cache,
                          const double *v_cache, const int32_t *row, int L,
                          int kvh, int num_kv_heads, int head_dim,
                          int block_size)
{
    for (int t = 0; t < L; ++t) {
        int block = row[t / block_size];
        int offset = t % block_size;
        size_t src = pool_row(block, kvh, offset, num_kv_heads, block_size,
                              head_dim);
        memcpy(K + (size_t)t * head_dim, k_cache + src,
               sizeof(double) * head_dim);
        memcpy(V + (size_t)t * head_dim, v_cache + src,
               sizeof(double) * head_dim);
    }
}

/* Dense attention of one query over L contiguous keys/values:
 *   z_t = scale * q . K_t,  w_t = exp(z_t - max z),  out = sum_t w_t V_t / sum_t w_t.
 * [P3] §1.3 (softmax(Q K^T / sqrt(d)) V over the first t tokens);
 * [P4] §3.1 compute_attention (gather, then the same dense softmax).
 * L == 0 writes zeros (the pages define no result for an empty context). */
static void dense_attention(double *out, const double *q, const double *K,
                            const double *V, double *z, int L, int head_dim,
                            double scale)
{
    for (int d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (L == 0)
        return;
    double m = -INFINITY;
    for (int t = 0; t < L; ++t) {
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += q[d] * K[(size_t)t * head_dim + d];
        z[t] = scale * dot;
        if (z[t] > m)
            m = z[t];
    }
    double denom = 0.0;
    for (int t = 0; t < L; ++t) {
        double w = exp(z[t] - m);
        denom += w;
        for (int d = 0; d < head_dim; ++d)
            out[d] += w * V[(size_t)t * head_dim + d];
    }
    for (int d = 0; d < head_dim; ++d)
        out[d] /= denom;
}

/* Paged decode: for every sequence s and query head h, attention of
 * query[s, h] over the sequence's context_lens[s] cached tokens, gathered
 * through its block table. Query head h reads kv head h / (num_heads /
 * num_kv_heads) (contiguous GQA groups; the pages leave GQA open, [P3] §10).
 * [P4] §3.1 (gather-then-attend); [P5] §3.2 (the operation's inputs:
 * query, key_cache, value_cache, block_tables, context_lens, scale). */
int oracle_paged_decode(double *out, const double *query,
                        const double *k_cache, const double *v_cache,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs,
                        int num_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, double scale)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        head_dim <= 0 || block_size <= 0 || num_blocks < 0 ||
        num_heads % num_kv_heads != 0)
        return OR_BAD_ARG;
    int group = num_heads / num_kv_heads;
    int max_len = 0;
    for (int s = 0; s < num_seqs; ++s) {
        if (context_lens[s] < 0)
            return OR_BAD_ARG;
        int rc = check_table_row(block_tables + (size_t)s * max_blocks_per_seq,
                                 context_lens[s], block_size,
                                 max_blocks_per_seq, num_blocks);
        if (rc != OR_OK)
            return rc;
        if (context_lens[s] > max_len)
            max_len = context_lens[s];
    }
    size_t n = (size_t)(max_len > 0 ? max_len : 1);
    double *K = malloc(sizeof(double) * n * head_dim);
    double *V = malloc(sizeof(double) * n * head_dim);
    double *z = malloc(sizeof(double) * n);
    if (!K || !V || !z) {
        free(K); free(V); free(z);
        return OR_NO_MEMORY;
    }
    for (int s = 0; s < num_seqs; ++s) {
        const int32_t *row = block_tables + (size_t)s * max_blocks_per_seq;
        int L = context_lens[s];
        for (int h = 0; h < num_heads; ++h) {
            int kvh = h / group;
            gather_tokens(K, V, k_cache, v_cache, row, L, kvh, num_kv_heads,
                          head_dim, block_size);
            size_t qo = ((size_t)s * num_heads + h) * head_dim;
            dense_attention(out + qo, query + qo, K, V, z, L, head_dim, scale);
        }
    }
    free(K); free(V); free(z);
    return OR_OK;
}

/* Split-K partials. Partition p of sequence s covers tokens
 * [p * P, min((p + 1) * P, L)). For each (s, h, p) with a non-empty range:
 *   m_p   = max_t z_t
 *   l_p   = sum_t exp(z_t - m_p)
 *   acc_p = sum_t exp(z_t - m_p) V_t              (unnormalised)
 * The pages only name the partitioned (V2) kernel for few, long sequences
 * ([P5] §2.3); the partial triple is the standard log-sum-exp split of the
 * dense softmax above. Layout: part_m/part_l [num_seqs, num_heads, max_parts],
 * part_acc [num_seqs, num_heads, max_parts, head_dim]. Entries of empty
 * partitions are left untouched. */
int oracle_splitk_partials(double *part_m, double *part_l, double *part_acc,
                           const double *query, const double *k_cache,
                           const double *v_cache, const int32_t *block_tables,
                           int max_blocks_per_seq, const int32_t *context_lens,
                           int num_seqs, int num_heads, int num_kv_heads,
                           int head_dim, int block_size, int num_blocks,
                           double scale, int partition_size, int max_parts)
{
    if (partition_size <= 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0)
        return OR_BAD_ARG;
    int group = num_heads / num_kv_heads;
    int max_len = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        if (L < 0)
            return OR_BAD_ARG;
        int rc = check_table_row(block_tables + (size_t)s * max_blocks_per_seq,
                                 L, block_size, max_blocks_per_seq, num_blocks);
        if (rc != OR_OK)
            return rc;
        if ((L + partition_size - 1) / partition_size > max_parts)
            return OR_BAD_ARG;
        if (L > max_len)
            max_len = L;
    }
    size_t n = (size_t)(max_len > 0 ? max_len : 1);
    double *K = malloc(sizeof(double) * n * head_dim);
    double *V = malloc(sizeof(double) * n * head_dim);
    if (!K || !V) {
        free(K); free(V);
        return OR_NO_MEMORY;
    }
    for (int s = 0; s < num_seqs; ++s) {
        const int32_t *row = block_tables + (size_t)s * max_blocks_per_seq;
        int L = context_lens[s];
        int nparts = (L + partition_size - 1) / partition_size;
        for (int h = 0; h < num_heads; ++h) {
            gather_tokens(K, V, k_cache, v_cache, row, L, h / group,
                          num_kv_heads, head_dim, block_size);
            const double *q = query + ((size_t)s * num_heads + h) * head_dim;
            for (int p = 0; p < nparts; ++p) {
                int t0 = p * partition_size;
                int t1 = t0 + partition_size < L ? t0 + partition_size : L;
                size_t idx = ((size_t)s * num_heads + h) * max_parts + p;
                double *acc = part_acc + idx * head_dim;
                double m = -INFINITY;
                for (int t = t0; t < t1; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += q[d] * K[(size_t)t * head_dim + d];
                    if (scale * dot > m)
                        m = scale * dot;
                }
                double l = 0.0;
                for (int d = 0; d < head_dim; ++d)
                    acc[d] = 0.0;
                for (int t = t0; t < t1; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += q[d] * K[(size_t)t * head_dim + d];
                    double w = exp(scale * dot - m);
                    l += w;
                    for (int d = 0; d < head_dim; ++d)
                        acc[d] += w * V[(size_t)t * head_dim + d];
                }
                part_m[idx] = m;
                part_l[idx] = l;
            }
        }
    }
    free(K); free(V);
    return OR_OK;
}

/* Log-sum-exp merge of split-K partials (closed form):
 *   M = max_p m_p,  out = sum_p e^(m_p - M) acc_p / sum_p e^(m_p - M) l_p
 * over the ceil(L / P) partitions of each sequence; L == 0 writes zeros. */
int oracle_splitk_merge(double *out, const double *part_m,
                        const double *part_l, const double *part_acc,
                        const int32_t *context_lens, int num_seqs,
                        int num_heads, int head_dim, int partition_size,
                        int max_parts)
{
    if (partition_size <= 0 || head_dim <= 0 || num_heads <= 0)
        return OR_BAD_ARG;
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        if (L < 0)
            return OR_BAD_ARG;
        int nparts = (L + partition_size - 1) / partition_size;
        if (nparts > max_parts)
            return OR_BAD_ARG;
        for (int h = 0; h < num_heads; ++h) {
            size_t base = ((size_t)s * num_heads + h) * max_parts;
            double *o = out + ((size_t)s * num_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            if (nparts == 0)
                continue;
            double M = -INFINITY;
            for (int p = 0; p < nparts; ++p)
                if (part_m[base + p] > M)
                    M = part_m[base + p];
            double denom = 0.0;
            for (int p = 0; p < nparts; ++p) {
                double w = exp(part_m[base + p] - M);
                denom += w * part_l[base + p];
                for (int d = 0; d < head_dim; ++d)
                    o[d] += w * part_acc[(base + p) * head_dim + d];
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= denom;
        }
    }
    return OR_OK;
}

/* Slot write: token i's key and value rows, for every kv head h, go to
 * physical block slot / block_size at offset slot % block_size, as raw bytes.
 * Tokens are applied in order; a negative slot is skipped.
 * [P3] §3.1 (slot_mapping maps a token to (block_id, offset)) and §4.2
 * (block_id = slot / block_size, offset = slot % block_size); [P4] §3.4
 * (the runner writes each new token's K/V into its block). */
int oracle_reshape_and_cache(unsigned char *k_cache, unsigned char *v_cache,
                             const unsigned char *key,
                             const unsigned char *value,
                             const int32_t *slot_mapping, int num_tokens,
                             int num_blocks, int num_kv_heads, int head_dim,
                             int block_size, int elt_bytes)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || elt_bytes <= 0)
        return OR_BAD_ARG;
    size_t row_bytes = (size_t)head_dim * elt_bytes;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size)
            return OR_BAD_SLOT;
        int block = (int)(slot / block_size);
        int offset = (int)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t dst = pool_row(block, h, offset, num_kv_heads, block_size,
                                  head_dim) * elt_bytes;
            size_t src = ((size_t)i * num_kv_heads + h) * row_bytes;
            memcpy(k_cache + dst, key + src, row_bytes);
            memcpy(v_cache + dst, value + src, row_bytes);
        }
    }
    return OR_OK;
}

/* Copy-on-write block copy: for each pair (src, dst), the whole physical
 * block dst of both pools becomes a byte copy of block src ([P4] §3.3: the
 * new block receives all of the old block's contents by a device-to-device
 * copy). Pairs are applied in order. */
int oracle_copy_blocks(unsigned char *k_cache, unsigned char *v_cache,
                       const int64_t *src_dst_pairs, int num_pairs,
                       int num_blocks, int64_t block_bytes)
{
    if (num_pairs < 0 || block_bytes <= 0)
        return OR_BAD_ARG;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = src_dst_pairs[2 * i];
        int64_t dst = src_dst_pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return OR_BAD_BLOCK_ID;
        memmove(k_cache + dst * block_bytes, k_cache + src * block_bytes,
                (size_t)block_bytes);
        memmove(v_cache + dst * block_bytes, v_cache + src * block_bytes,
                (size_t)block_bytes);
    }
    return OR_OK;
}

/* Paged prefill (chunked prefill) attention. Sequence s has
 * q_len_s = q_start[s + 1] - q_start[s] new query tokens, rows q_start[s] ..
 * of query/out, already written into its cache; query token i sits at
 * position pos = context_lens[s] - q_len_s + i and attends to the cache
 * tokens 0 .. pos (causal): out = softmax(scale q . K_t) V over t <= pos.
 * Decode is the case q_len_s = 1. The pages place prefill beside decode in
 * the serving step ([P4] §3.4, the model forward over the new tokens) and
 * give the kernel a num_tokens axis of queries ([P3] §3.1, PagedAttnParams).
 * Requires q_len_s <= context_lens[s]. */
int oracle_paged_prefill(double *out, const double *query, const int32_t *q_start,
                         const double *k_cache, const double *v_cache,
                         const int32_t *block_tables, int max_blocks_per_seq,
                         const int32_t *context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, double scale)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_heads % num_kv_heads != 0)
        return OR_BAD_ARG;
    int group = num_heads / num_kv_heads;
    int max_len = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int L = context_lens[s];
        int ql = q_start[s + 1] - q_start[s];
        if (L < 0 || ql < 0 || ql > L)
            return OR_BAD_ARG;
        int rc = check_table_row(block_tables + (size_t)s * max_blocks_per_seq, L,
                                 block_size, max_blocks_per_seq, num_blocks);
        if (rc != OR_OK)
            return rc;
        if (L > max_len)
            max_len = L;
    }
    size_t n = (size_t)(max_len > 0 ? max_len : 1);
    double *K = malloc(sizeof(double) * n * head_dim);
    double *V = malloc(sizeof(double) * n * head_dim);
    double *z = malloc(sizeof(double) * n);
    if (!K || !V || !z) {
        free(K); free(V); free(z);
        return OR_NO_MEMORY;
    }
    for (int s = 0; s < num_seqs; ++s) {
        const int32_t *row = block_tables + (size_t)s * max_blocks_per_seq;
        int L = context_lens[s];
        int ql = q_start[s + 1] - q_start[s];
        for (int h = 0; h < num_heads; ++h) {
            gather_tokens(K, V, k_cache, v_cache, row, L, h / group, num_kv_heads,
                          head_dim, block_size);
            for (int i = 0; i < ql; ++i) {
                int pos = L - ql + i;
                size_t qo = ((size_t)(q_start[s] + i) * num_heads + h) * head_dim;
                dense_attention(out + qo, query + qo, K, V, z, pos + 1, head_dim, scale);
            }
        }
    }
    free(K); free(V); free(z);
    return OR_OK;
}

/* ------------------------------------------------------------ int8 KV cache
 *
 * The pages list int8 among the paged backend's storage types ([P4] §3.4,
 * attention backends) and name KV quantization as a way to cut cache memory
 * at some cost in precision ([P2] §2.3, §6.3); they give no scheme. Reading
 * taken here: symmetric int8 per (token, kv head) row of head_dim values,
 * one fp32 scale per row, decided when the row is written:
 *     amax = max_d |x_d|,  inv = 127 / amax,  q_d = round_half_even(x_d * inv)
 *     clamped to [-127, 127],  scale = amax / 127;  amax = 0 gives q = 0, scale 0.
 * Every step is one IEEE fp32 operation (x is the stored 16- or 32-bit value,
 * exact in fp32), so the integer codes are the same wherever this is run in
 * fp32 with round-to-nearest. The cache then holds K_t = q_t * scale_t.
 * Scale pools: [num_blocks, num_kv_heads, block_size] fp32. */

static void quantize_row(const float *x, int n, int8_t *q, float *scale)
{
    float amax = 0.0f;
    for (int d = 0; d < n; ++d) {
        float a = fabsf(x[d]);
        if (a > amax)
            amax = a;
    }
    if (amax == 0.0f) {
        for (int d = 0; d < n; ++d)
            q[d] = 0;
        *scale = 0.0f;
        return;
    }
    float inv = 127.0f / amax;
    for (int d = 0; d < n; ++d) {
        float y = x[d] * inv;
        long r = lrintf(y);
        if (r > 127)
            r = 127;
        if (r < -127)
            r = -127;
        q[d] = (int8_t)r;
    }
    *scale = amax / 127.0f;
}

/* rows x n values -> rows x n codes and rows scales. */
int oracle_quantize_rows(const float *x, int rows, int n, int8_t *q, float *scale)
{
    if (rows < 0 || n <= 0)
        return OR_BAD_ARG;
    for (int r = 0; r < rows; ++r)
        quantize_row(x + (size_t)r * n, n, q + (size_t)r * n, scale + r);
    return OR_OK;
}

/* Slot write into an int8 cache: token i's row for kv head h is quantized
 * and lands at (slot / block_size, h, slot % block_size) of the code pools,
 * its scale at the same (block, h, offset) of the scale pools. slot < 0 is
 * skipped. key/value: [num_tokens, num_kv_heads, head_dim] fp32 (the stored
 * values, widened). */
int oracle_reshape_and_cache_q8(int8_t *k_cache, int8_t *v_cache, float *k_scale, float *v_scale,
                                const float *key, const float *value, const int32_t *slot_mapping,
                                int num_tokens, int num_blocks, int num_kv_heads, int head_dim,
                                int block_size)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
        return OR_BAD_ARG;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size)
            return OR_BAD_SLOT;
        int block = (int)(slot / block_size);
        int offset = (int)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            size_t row = pool_row(block, h, offset, num_kv_heads, block_size, head_dim);
            size_t srow = ((size_t)block * num_kv_heads + h) * block_size + offset;
            size_t src = ((size_t)i * num_kv_heads + h) * head_dim;
            quantize_row(key + src, head_dim, k_cache + row, k_scale + srow);
            quantize_row(value + src, head_dim, v_cache + row, v_scale + srow);
        }
    }
    return OR_OK;
}
