/*
 * pa_oracle.c -- plain, slow fp64 CPU oracle for attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load the library built from this file.
 * The product path never calls it and shares no code with it.
 *
 * What it follows (source pages, by title and section):
 *
 *  [KV]  "Inference optimization" (AI Engineering from Scratch, Phase 10 / 12),
 *        section "KV cache" and "Build it -- Step 1: a KV cache from scratch":
 *        the new token's K and V rows are written into the cache first, and
 *        attention then reads every cached row including the new one
 *        ("token 5: compute K5, V5, read K1-4, V1-4 from the cache").
 *  [SDPA] same page, "Step 2: attention with the KV cache": scores are
 *        q . K^T / sqrt(d) (here: times a caller-given scale), the row maximum
 *        is subtracted, the scores are exponentiated and normalised by their
 *        sum, and the weights multiply V.  A block of Lq query rows placed at
 *        the end of Lk keys is masked so that query row i sees the keys
 *        j <= i + (Lk - Lq) (the mask is aligned to the bottom-right corner).
 *  [PAGE] "vLLM serving internals" (Phase 17 / 04), "PagedAttention as a
 *        virtual memory system" and "Key terms"; "Inference optimization",
 *        "Paged attention": the cache is split into fixed-size physical blocks
 *        and a per-sequence block table maps each logical token position to a
 *        physical block ID.
 *
 * Every function here is the definition written out, in fp64, with libm exp.
 * There is no blocking, no online softmax, no split of the key range.
 *
 * Data layouts (the same ones the library's boundary uses):
 *   q, out        [num_q_tokens, num_q_heads, head_dim]       (q: bf16 bits)
 *   k/v cache     [num_blocks, num_kv_heads, block_size, head_dim] bf16 bits
 *   block_tables  [num_seqs, max_blocks_per_seq] int32, -1 = unused entry
 *   context_lens  [num_seqs] int32, including this step's new tokens
 *   query_start   [num_seqs + 1] int32 prefix offsets of each sequence's rows
 *   slot_mapping  [num_new_tokens] int32, slot = block * block_size + offset,
 *                 negative = padding row, not written
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/*
 * ORACLE_MUTATION (test-only builds): each value plants one plausible mistake so
 * that the pin tests can show they catch it.  The default build has none.
 *   1: the newest key is dropped (mask one short)     2: KV head = h % Hkv
 *   3: the scale is ignored                          4: cache rows read head-major
 *   5: no normalisation by the weight sum            6: no max subtraction
 *   7: the append writes every head's row to head 0  8: offset = pos / block_size
 *   FP8 (E4M3) cache:
 *   9: exponent bias 8 when decoding                 10: encoding rounds toward zero
 *  11: encoding does not saturate at 448            12: attention leaves out the V scale
 *  13: the append multiplies by the scale, not by its inverse
 */
#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_SHAPE (-2)
#define ORACLE_ERR_RANGE (-5)
#define ORACLE_ERR_NOMEM (-8)

/* bf16 is the upper half of an IEEE binary32; widening to double is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Physical location of logical token `pos` of sequence `s` [PAGE]:
 * block ID = table[s][pos / block_size], offset = pos % block_size.
 * Returns -1 when the table entry is missing or out of the pool.
 */
static long long physical_row(const int32_t *block_tables, int max_blocks, int s,
                              int pos, int block_size, int num_blocks)
{
    int logical_block = pos / block_size;
    if (logical_block >= max_blocks)
        return -1;
    int32_t phys = block_tables[(long long)s * max_blocks + logical_block];
    if (phys < 0 || phys >= num_blocks)
        return -1;
#if ORACLE_MUTATION == 8
    return (long long)phys * block_size + (pos / block_size) % block_size;
#else
    return (long long)phys * block_size + (pos % block_size);
#endif
}

/*
 * Slot of every new token [PAGE]: for sequence s with query rows
 * query_start[s] .. query_start[s+1]-1, row i sits at logical position
 * context_lens[s] - qlen + i and goes to slot table[s][pos/bs]*bs + pos%bs.
 */
int oracle_slot_mapping(int32_t *slot_out, const int32_t *block_tables, int max_blocks,
                        const int32_t *context_lens, const int32_t *query_start,
                        int num_seqs, int block_size, int num_blocks)
{
    for (int s = 0; s < num_seqs; ++s) {
        int q0 = query_start[s], qlen = query_start[s + 1] - query_start[s];
        for (int i = 0; i < qlen; ++i) {
            int pos = context_lens[s] - qlen + i;
            if (pos < 0)
                return ORACLE_ERR_SHAPE;
            long long row = physical_row(block_tables, max_blocks, s, pos, block_size, num_blocks);
            if (row < 0)
                return ORACLE_ERR_RANGE;
            slot_out[q0 + i] = (int32_t)row;
        }
    }
    return ORACLE_OK;
}

/*
 * Cache append [KV]: copy row t of k_new / v_new (every KV head) into slot
 * slot_mapping[t]; negative slots are padding and are skipped.  A byte copy.
 */
int oracle_cache_append(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                        uint16_t *v_cache, const int32_t *slot_mapping, int num_tokens,
                        int num_blocks, int num_kv_heads, int head_dim, int block_size)
{
    long long num_slots = (long long)num_blocks * block_size;
    for (int t = 0; t < num_tokens; ++t) {
        long long slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_slots)
            return ORACLE_ERR_RANGE;
        long long blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
#if ORACLE_MUTATION == 7
            long long dst = ((blk * num_kv_heads + 0) * block_size + off) * head_dim;
#else
            long long dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
#endif
            long long src = ((long long)t * num_kv_heads + h) * head_dim;
            memcpy(k_cache + dst, k_new + src, (size_t)head_dim * sizeof(uint16_t));
            memcpy(v_cache + dst, v_new + src, (size_t)head_dim * sizeof(uint16_t));
        }
    }
    return ORACLE_OK;
}

/*
 * One output row [SDPA] over keys 0..last_key of sequence s, for query head h
 * which reads KV head kvh.  scores[j] = scale * sum_d q[d] * K_j[d]; m = max_j
 * scores[j]; w_j = exp(scores[j] - m); out = sum_j w_j V_j / sum_j w_j.
 * The sum is built in `acc` (head_dim doubles) and only then stored, so two
 * calls for the same row write the same values.
 */
static int attend_one(double *out, const uint16_t *q_row, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *block_tables, int max_blocks,
                      int s, int last_key, int kvh, int num_kv_heads, int head_dim,
                      int block_size, int num_blocks, double scale, double *scores, double *acc)
{
#if ORACLE_MUTATION == 1
    int nkeys = last_key;
#else
    int nkeys = last_key + 1;
#endif
#if ORACLE_MUTATION == 3
    scale = 1.0;
#endif
    for (int d = 0; d < head_dim; ++d)
        acc[d] = 0.0;
    if (nkeys <= 0) {
        memcpy(out, acc, sizeof(double) * (size_t)head_dim);
        return ORACLE_OK; /* softmax over an empty set: the output is defined as zeros */
    }

    double m = -INFINITY;
    for (int j = 0; j < nkeys; ++j) {
        long long row = physical_row(block_tables, max_blocks, s, j, block_size, num_blocks);
        if (row < 0)
            return ORACLE_ERR_RANGE;
        long long blk = row / block_size, off = row % block_size;
#if ORACLE_MUTATION == 4
        const uint16_t *krow = k_cache + ((blk * block_size + off) * num_kv_heads + kvh) * head_dim;
#else
        const uint16_t *krow = k_cache + ((blk * num_kv_heads + kvh) * block_size + off) * head_dim;
#endif
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += bf16_bits_to_double(q_row[d]) * bf16_bits_to_double(krow[d]);
        scores[j] = scale * dot;
        if (scores[j] > m)
            m = scores[j];
    }
    double denom = 0.0;
    for (int j = 0; j < nkeys; ++j) {
#if ORACLE_MUTATION == 6
        double w = exp(scores[j]);
#else
        double w = exp(scores[j] - m);
#endif
        long long row = physical_row(block_tables, max_blocks, s, j, block_size, num_blocks);
        long long blk = row / block_size, off = row % block_size;
        const uint16_t *vrow = v_cache + ((blk * num_kv_heads + kvh) * block_size + off) * head_dim;
        for (int d = 0; d < head_dim; ++d)
            acc[d] += w * bf16_bits_to_double(vrow[d]);
        denom += w;
    }
#if ORACLE_MUTATION != 5
    for (int d = 0; d < head_dim; ++d)
        acc[d] /= denom;
#else
    (void)denom;
#endif
    memcpy(out, acc, sizeof(double) * (size_t)head_dim);
    return ORACLE_OK;
}

/*
 * Attention of every query row of a varlen batch over its paged cache.
 * Row i of sequence s (0 <= i < qlen) is at position p = ctx - qlen + i and
 * sees keys 0..p [SDPA mask].  Query head h reads KV head h / (Hq / Hkv)
 * (consecutive query heads share a KV head).  Decode is the case qlen = 1.
 * If `only_rows` is non-NULL, only the listed (token, head) pairs are
 * computed (n_only of them); the other outputs are left untouched.
 */
int oracle_paged_attention(double *out, const uint16_t *q, const uint16_t *k_cache,
                           const uint16_t *v_cache, const int32_t *block_tables,
                           int max_blocks, const int32_t *context_lens,
                           const int32_t *query_start, int num_seqs, int num_q_heads,
                           int num_kv_heads, int head_dim, int block_size, int num_blocks,
                           double scale, const int32_t *only_rows, int n_only)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return ORACLE_ERR_SHAPE;
    int group = num_q_heads / num_kv_heads;
    int num_tokens = query_start[num_seqs];
    int max_ctx = 0;
    for (int s = 0; s < num_seqs; ++s)
        if (context_lens[s] > max_ctx)
            max_ctx = context_lens[s];

    /* Flatten the work into (token, head) items; token -> sequence lookup. */
    int32_t *seq_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)(num_tokens > 0 ? num_tokens : 1));
    if (!seq_of)
        return ORACLE_ERR_NOMEM;
    for (int s = 0; s < num_seqs; ++s)
        for (int t = query_start[s]; t < query_start[s + 1]; ++t)
            seq_of[t] = s;
    long long n_items = only_rows ? n_only : (long long)num_tokens * num_q_heads;

    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(max_ctx > 0 ? max_ctx : 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)head_dim);
        if (!scores || !acc) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (long long it = 0; it < n_items; ++it) {
            if (!scores || !acc)
                continue;
            int t, h;
            if (only_rows) {
                t = only_rows[2 * it];
                h = only_rows[2 * it + 1];
            } else {
                t = (int)(it / num_q_heads);
                h = (int)(it % num_q_heads);
            }
            int s = seq_of[t];
            int qlen = query_start[s + 1] - query_start[s];
            int pos = context_lens[s] - qlen + (t - query_start[s]);
            int rc = attend_one(out + ((long long)t * num_q_heads + h) * head_dim,
                                q + ((long long)t * num_q_heads + h) * head_dim, k_cache,
                                v_cache, block_tables, max_blocks, s, pos,
#if ORACLE_MUTATION == 2
                                h % num_kv_heads,
#else
                                h / group,
#endif
                                num_kv_heads, head_dim, block_size, num_blocks, scale, scores, acc);
            if (rc != ORACLE_OK) {
#pragma omp atomic write
                status = rc;
            }
        }
        free(scores);
        free(acc);
    }
    free(seq_of);
    return status;
}

/*
 * ---- FP8 KV cache -------------------------------------------------------
 *
 * The pages serve Llama 3.3 70B in FP8 ("vLLM serving internals",
 * introduction and "Numbers to remember"; "How vLLM gets real throughput on
 * H100s", "Hopper-specific tunings") without fixing a format.  The reading
 * taken here: the cache stores E4M3 codes of the OCP 8-bit floating point
 * specification ("FN" variant: sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 = NaN, largest finite 1.75 * 2^8 = 448,
 * subnormals m/8 * 2^-6) with one scale per tensor: code = E4M3(x * (1/scale))
 * rounded to nearest-even and saturated to +-448, value = E4M3value * scale.
 */
double oracle_e4m3_to_f64(uint8_t c)
{
    int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
#if ORACLE_MUTATION == 9
    double v = (e == 0) ? ldexp(m / 8.0, -7) : ldexp(1.0 + m / 8.0, e - 8);
#else
    double v = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
#endif
    return sgn ? -v : v;
}

uint8_t oracle_f32_to_e4m3(float xf)
{
    double x = xf; /* exact */
    if (isnan(x))
        return 0x7F;
    uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isinf(a))
        return (uint8_t)(sgn | 0x7E);
    if (a == 0.0)
        return sgn;
    int e2;
    frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1): floor(log2 a) = e2 - 1 */
    int ex = e2 - 1;
    double quantum = ex < -6 ? ldexp(1.0, -9) : ldexp(1.0, ex - 3);
#if ORACLE_MUTATION == 10
    double r = floor(a / quantum) * quantum;
#else
    double r = nearbyint(a / quantum) * quantum; /* a / quantum is exact; ties to even */
#endif
#if ORACLE_MUTATION != 11
    if (r > 448.0)
        r = 448.0; /* saturate to the largest finite value */
#endif
    if (r == 0.0)
        return sgn;
    frexp(r, &e2);
    ex = e2 - 1;
    if (ex < -6) /* subnormal: exponent field 0, r = m * 2^-9 */
        return (uint8_t)(sgn | (uint8_t)(r / ldexp(1.0, -9)));
    int m = (int)((r / ldexp(1.0, ex) - 1.0) * 8.0);
    return (uint8_t)(sgn | (uint8_t)((ex + 7) << 3) | (uint8_t)m);
}

/*
 * FP8 cache append [KV]: for every token with slot >= 0 and every KV head,
 * code = E4M3(bf16 value * inv_scale), the product taken in binary32.
 */
int oracle_cache_append_fp8(const uint16_t *k_new, const uint16_t *v_new, uint8_t *k_cache, uint8_t *v_cache,
                            const int32_t *slot_mapping, int num_tokens, int num_blocks, int num_kv_heads,
                            int head_dim, int block_size, float k_inv_scale, float v_inv_scale)
{
    long long num_slots = (long long)num_blocks * block_size;
    for (int t = 0; t < num_tokens; ++t) {
        long long slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_slots)
            return ORACLE_ERR_RANGE;
        long long blk = slot / block_size, off = slot % block_size;
        for (int h = 0; h < num_kv_heads; ++h) {
            long long dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
            long long src = ((long long)t * num_kv_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d) {
#if ORACLE_MUTATION == 13
                float kx = (float)bf16_bits_to_double(k_new[src + d]) * (1.0f / k_inv_scale);
                float vx = (float)bf16_bits_to_double(v_new[src + d]) * (1.0f / v_inv_scale);
#else
                float kx = (float)bf16_bits_to_double(k_new[src + d]) * k_inv_scale;
                float vx = (float)bf16_bits_to_double(v_new[src + d]) * v_inv_scale;
#endif
                k_cache[dst + d] = oracle_f32_to_e4m3(kx);
                v_cache[dst + d] = oracle_f32_to_e4m3(vx);
            }
        }
    }
    return ORACLE_OK;
}

/* One output row [SDPA] over an FP8 cache: K_j = E4M3value * k_scale, V_j likewise. */
static int attend_one_fp8(double *out, const uint16_t *q_row, const uint8_t *k_cache, const uint8_t *v_cache,
                          const int32_t *block_tables, int max_blocks, int s, int last_key, int kvh,
                          int num_kv_heads, int head_dim, int block_size, int num_blocks, double scale,
                          double k_scale, double v_scale, double *scores, double *acc)
{
    int nkeys = last_key + 1;
    for (int d = 0; d < head_dim; ++d)
        acc[d] = 0.0;
    if (nkeys <= 0) {
        memcpy(out, acc, sizeof(double) * (size_t)head_dim);
        return ORACLE_OK;
    }
    double m = -INFINITY;
    for (int j = 0; j < nkeys; ++j) {
        long long row = physical_row(block_tables, max_blocks, s, j, block_size, num_blocks);
        if (row < 0)
            return ORACLE_ERR_RANGE;
        long long blk = row / block_size, off = row % block_size;
        const uint8_t *krow = k_cache + ((blk * num_kv_heads + kvh) * block_size + off) * head_dim;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += bf16_bits_to_double(q_row[d]) * (oracle_e4m3_to_f64(krow[d]) * k_scale);
        scores[j] = scale * dot;
        if (scores[j] > m)
            m = scores[j];
    }
    double denom = 0.0;
    for (int j = 0; j < nkeys; ++j) {
        double w = exp(scores[j] - m);
        long long row = physical_row(block_tables, max_blocks, s, j, block_size, num_blocks);
        long long blk = row / block_size, off = row % block_size;
        const uint8_t *vrow = v_cache + ((blk * num_kv_heads + kvh) * block_size + off) * head_dim;
        for (int d = 0; d < head_dim; ++d)
#if ORACLE_MUTATION == 12
            acc[d] += w * oracle_e4m3_to_f64(vrow[d]);
#else
            acc[d] += w * (oracle_e4m3_to_f64(vrow[d]) * v_scale);
#endif
        denom += w;
    }
    for (int d = 0; d < head_dim; ++d)
        acc[d] /= denom;
    memcpy(out, acc, sizeof(double) * (size_t)head_dim);
    return ORACLE_OK;
}

/* oracle_paged_attention over an FP8 cache (same conventions). */
int oracle_paged_attention_fp8(double *out, const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                               const int32_t *block_tables, int max_blocks, const int32_t *context_lens,
                               const int32_t *query_start, int num_seqs, int num_q_heads, int num_kv_heads,
                               int head_dim, int block_size, int num_blocks, double scale, double k_scale,
                               double v_scale, const int32_t *only_rows, int n_only)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return ORACLE_ERR_SHAPE;
    int group = num_q_heads / num_kv_heads;
    int num_tokens = query_start[num_seqs];
    int max_ctx = 0;
    for (int s = 0; s < num_seqs; ++s)
        if (context_lens[s] > max_ctx)
            max_ctx = context_lens[s];
    int32_t *seq_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)(num_tokens > 0 ? num_tokens : 1));
    if (!seq_of)
        return ORACLE_ERR_NOMEM;
    for (int s = 0; s < num_seqs; ++s)
        for (int t = query_start[s]; t < query_start[s + 1]; ++t)
            seq_of[t] = s;
    long long n_items = only_rows ? n_only : (long long)num_tokens * num_q_heads;
    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(max_ctx > 0 ? max_ctx : 1));
        double *acc = (double *)malloc(sizeof(double) * (size_t)head_dim);
        if (!scores || !acc) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (long long it = 0; it < n_items; ++it) {
            if (!scores || !acc)
                continue;
            int t, h;
            if (only_rows) {
                t = only_rows[2 * it];
                h = only_rows[2 * it + 1];
            } else {
                t = (int)(it / num_q_heads);
                h = (int)(it % num_q_heads);
            }
            int s = seq_of[t];
            int qlen = query_start[s + 1] - query_start[s];
            int pos = context_lens[s] - qlen + (t - query_start[s]);
            int rc = attend_one_fp8(out + ((long long)t * num_q_heads + h) * head_dim,
                                    q + ((long long)t * num_q_heads + h) * head_dim, k_cache, v_cache, block_tables,
                                    max_blocks, s, pos, h / group, num_kv_heads, head_dim, block_size, num_blocks,
                                    scale, k_scale, v_scale, scores, acc);
            if (rc != ORACLE_OK) {
#pragma omp atomic write
                status = rc;
            }
        }
        free(scores);
        free(acc);
    }
    free(seq_of);
    return status;
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
