/*
 * CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library; the product path never does.  It shares
 * no code with the CUDA library.
 *
 * What it computes (the plain definition, no blocking or fusion):
 *
 *   Block table translation -- a sequence's token t lives in logical block
 *   t / block_size at offset t % block_size; the block table maps the
 *   logical block to a physical block of the shared pool
 *   (openeuler.csdn.net PagedAttention explainer, section 4.2; aiknowledge.cn
 *   "2.2 PagedAttention 与 KV Cache 分页管理", section 2.2.3 worked example).
 *
 *   Pool layout -- pool[block][kv_head][offset][d], row-major.
 *
 *   Decode attention for sequence s and query head h (one query token):
 *     g   = h / (Hq / Hkv)               (consecutive query heads share a kv head)
 *     x_t = scale * sum_d q[s,h,d] * K[slot(s,t), g, d],  t = 0 .. L-1
 *     out = sum_t exp(x_t - max x) V[slot(s,t), g, :] / sum_t exp(x_t - max x)
 *   with L = context_lens[s] tokens, no mask, and out = 0 when L = 0.  The
 *   pages give no formula; this is softmax(q K^T / sqrt(d)) V over the cached
 *   tokens, the plainest reading of "attention over the KV cache"
 *   (openeuler.csdn.net explainer, section 2.2).
 *
 * A chunk of new tokens per sequence (oracle_paged_attention_chunk): sequence s
 * owns query rows query_start[s] .. query_start[s+1]-1, which are the last
 * n_s tokens of its L_s cached tokens; row i (0-based) sits at position
 * L_s - n_s + i and attends causally to tokens 0 .. L_s - n_s + i -- each
 * token sees itself and what precedes it, as in autoregressive generation
 * (openeuler.csdn.net explainer, sections 2.1-2.2).  n_s = 1 is decode.
 *
 * Storage types are widened exactly to double: fp32 directly, bf16 by placing
 * its 16 bits on top of a float, fp16 by decoding sign/exponent/mantissa.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2, ORC_E4M3 = 3 };

/* FP8 E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; exponent 15 with mantissa 7 is NaN; largest finite 448). */
static double e4m3_value(uint8_t c) {
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

static double widen(const void *base, int64_t i, int dtype) {
    if (dtype == ORC_F32) return (double)((const float *)base)[i];
    if (dtype == ORC_E4M3) return e4m3_value(((const uint8_t *)base)[i]);
    uint16_t h = ((const uint16_t *)base)[i];
    if (dtype == ORC_BF16) {
        uint32_t u = (uint32_t)h << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    /* IEEE binary16 */
    int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 1024), e - 25);
    return sign ? -v : v;
}

/* Physical slot of token t of a sequence whose block table row is bt. */
int64_t oracle_slot(const int32_t *bt, int block_size, int64_t t) {
    return (int64_t)bt[t / block_size] * block_size + t % block_size;
}

/* Number of OpenMP threads a parallel region will get (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * out[i, :] (fp64, [n_items, D]) = attention for (items_s[i], items_h[i]).
 * Returns 0, or -1 on an index outside the given arrays (nothing written for
 * that item then), or -2 on bad shapes.
 */
/* Decode value of entry i of a K/V pool: code (or element) times its scale. */
static double pool_value(const void *pool, int64_t i, int kv_dtype, double kv_scale) {
    return widen(pool, i, kv_dtype) * kv_scale;
}

/*
 * Decode attention with K/V pools of their own element type: kv_dtype
 * ORC_E4M3 means FP8 codes, whose values are code value x k_scale (x
 * v_scale); for the other types the scales are 1.  q and out as in
 * oracle_paged_attention.
 */
int oracle_paged_attention_kv(double *out, const void *q, int q_dtype, const void *k_pool, const void *v_pool,
                              int kv_dtype, double k_scale, double v_scale, const int32_t *block_tables,
                              int max_blocks, const int32_t *context_lens, int S, int Hq, int Hkv, int D,
                              int block_size, int num_blocks, double scale, const int32_t *items_s,
                              const int32_t *items_h, int n_items, int num_threads);

int oracle_paged_attention(double *out, const void *q, const void *k_pool, const void *v_pool,
                           const int32_t *block_tables, int max_blocks,
                           const int32_t *context_lens, int S, int Hq, int Hkv, int D,
                           int block_size, int num_blocks, double scale, int dtype,
                           const int32_t *items_s, const int32_t *items_h, int n_items,
                           int num_threads) {
    return oracle_paged_attention_kv(out, q, dtype, k_pool, v_pool, dtype, 1.0, 1.0, block_tables, max_blocks,
                                     context_lens, S, Hq, Hkv, D, block_size, num_blocks, scale, items_s,
                                     items_h, n_items, num_threads);
}

int oracle_paged_attention_kv(double *out, const void *q, int q_dtype, const void *k_pool, const void *v_pool,
                              int kv_dtype, double k_scale, double v_scale, const int32_t *block_tables,
                              int max_blocks, const int32_t *context_lens, int S, int Hq, int Hkv, int D,
                              int block_size, int num_blocks, double scale, const int32_t *items_s,
                              const int32_t *items_h, int n_items, int num_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || block_size <= 0) return -2;
    int G = Hq / Hkv;
    int status = 0;
    if (num_threads <= 0) num_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(min : status)
    for (int i = 0; i < n_items; ++i) {
        int s = items_s[i], h = items_h[i];
        double *o = out + (int64_t)i * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (s < 0 || s >= S || h < 0 || h >= Hq) { status = -1; continue; }
        int g = h / G;
        int64_t L = context_lens[s];
        if (L <= 0) continue;
        if (L > (int64_t)max_blocks * block_size) { status = -1; continue; }
        const int32_t *bt = block_tables + (int64_t)s * max_blocks;
        int bad = 0;
        for (int64_t j = 0; j < (L + block_size - 1) / block_size; ++j)
            if (bt[j] < 0 || bt[j] >= num_blocks) bad = 1;
        if (bad) { status = -1; continue; }

        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        int64_t qbase = ((int64_t)s * Hq + h) * D;
        double mx = -INFINITY;
        for (int64_t t = 0; t < L; ++t) {
            int64_t slot = oracle_slot(bt, block_size, t);
            int64_t blk = slot / block_size, off = slot % block_size;
            int64_t kbase = ((blk * Hkv + g) * block_size + off) * D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += widen(q, qbase + d, q_dtype) * pool_value(k_pool, kbase + d, kv_dtype, k_scale);
            x[t] = scale * acc;
            if (x[t] > mx) mx = x[t];
        }
        double den = 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double w = exp(x[t] - mx);
            den += w;
            int64_t slot = oracle_slot(bt, block_size, t);
            int64_t blk = slot / block_size, off = slot % block_size;
            int64_t vbase = ((blk * Hkv + g) * block_size + off) * D;
            for (int d = 0; d < D; ++d) o[d] += w * pool_value(v_pool, vbase + d, kv_dtype, v_scale);
        }
        for (int d = 0; d < D; ++d) o[d] /= den;
        free(x);
    }
    return status;
}

/*
 * Causal attention of a chunk of query tokens per sequence (see the header).
 * out[i, :] (fp64, [n_items, D]) for (query row items_t[i], head items_h[i]).
 * Returns 0, -1 on an index outside the arrays, -2 on bad shapes.
 */
int oracle_paged_attention_chunk(double *out, const void *q, const void *k_pool, const void *v_pool,
                                 const int32_t *block_tables, int max_blocks, const int32_t *context_lens,
                                 const int32_t *query_start, int S, int T, int Hq, int Hkv, int D,
                                 int block_size, int num_blocks, double scale, int dtype,
                                 const int32_t *items_t, const int32_t *items_h, int n_items, int num_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || block_size <= 0) return -2;
    int G = Hq / Hkv;
    int status = 0;
    if (num_threads <= 0) num_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(min : status)
    for (int it = 0; it < n_items; ++it) {
        int t = items_t[it], h = items_h[it];
        double *o = out + (int64_t)it * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        if (t < 0 || t >= T || h < 0 || h >= Hq) { status = -1; continue; }
        int s = -1;
        for (int j = 0; j < S; ++j)
            if (query_start[j] <= t && t < query_start[j + 1]) s = j;
        if (s < 0) { status = -1; continue; }
        int64_t n = query_start[s + 1] - query_start[s];
        int64_t L = context_lens[s];
        if (n > L || L > (int64_t)max_blocks * block_size) { status = -1; continue; }
        int64_t upto = L - n + (t - query_start[s]) + 1; /* tokens this row sees */
        int g = h / G;
        const int32_t *bt = block_tables + (int64_t)s * max_blocks;
        int bad = 0;
        for (int64_t j = 0; j < (upto + block_size - 1) / block_size; ++j)
            if (bt[j] < 0 || bt[j] >= num_blocks) bad = 1;
        if (bad) { status = -1; continue; }
        double *x = (double *)malloc(sizeof(double) * (size_t)upto);
        int64_t qbase = ((int64_t)t * Hq + h) * D;
        double mx = -INFINITY;
        for (int64_t u = 0; u < upto; ++u) {
            int64_t slot = oracle_slot(bt, block_size, u);
            int64_t blk = slot / block_size, off = slot % block_size;
            int64_t kbase = ((blk * Hkv + g) * block_size + off) * D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += widen(q, qbase + d, dtype) * widen(k_pool, kbase + d, dtype);
            x[u] = scale * acc;
            if (x[u] > mx) mx = x[u];
        }
        double den = 0.0;
        for (int64_t u = 0; u < upto; ++u) {
            double w = exp(x[u] - mx);
            den += w;
            int64_t slot = oracle_slot(bt, block_size, u);
            int64_t blk = slot / block_size, off = slot % block_size;
            int64_t vbase = ((blk * Hkv + g) * block_size + off) * D;
            for (int d = 0; d < D; ++d) o[d] += w * widen(v_pool, vbase + d, dtype);
        }
        for (int d = 0; d < D; ++d) o[d] /= den;
        free(x);
    }
    return status;
}

/* Value of every E4M3 code (out[256]), for pinning against other decoders. */
void oracle_e4m3_table(double *out) {
    for (int c = 0; c < 256; ++c) out[c] = e4m3_value((uint8_t)c);
}
