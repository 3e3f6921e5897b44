/*
 * CPU oracle for one grouped-query-attention (GQA) decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path loads this file: only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may call it.  It shares no code, header,
 * table or helper with the CUDA library; inputs reach it as float64 host arrays.
 *
 * What it computes, and where that is stated:
 *
 *   - "GQA 阅读笔记" (zhongzhuzhou.org), section "GQA 架构", Algorithm 2 (GQA decode, step t,
 *     one layer): the G new key/value vectors of the step are written into the cache at row t,
 *     then every query head h looks up its group g(h) = ceil(h / (H/G)) (1-indexed), scores
 *     q_h against K_cache[:t+1, g] scaled by 1/sqrt(d_k), takes a softmax over those t+1
 *     scores and returns the weighted sum of V_cache[:t+1, g].
 *   - Same page, Algorithm 1 (MHA decode): the same step with one key/value head per query
 *     head; G = H reproduces it.
 *   - Lesson "r-tf2-gqa" (ttlab.hopto.org), sections on how the heads are grouped and what
 *     shrinks: query heads are grouped in contiguous blocks, and a grouped layer is run by
 *     repeating each key/value head for the query heads of its block and then running
 *     ordinary per-head attention ("expand then attend").
 *
 * The oracle follows that second form literally: expand_kv() materialises the repeated
 * key/value heads of one sequence, attend_one_head() is textbook single-head softmax attention.
 * Everything is float64, loops run in a fixed order, and there is no blocking, fusion or
 * online rescaling.  With 0-indexed heads the contiguous-block map is g(h) = floor(h / r),
 * r = H_q / H_kv, which is the 1-indexed ceil(h / (H/G)) of Algorithm 2 shifted by one.
 *
 * Readings where the pages leave a step open:
 *   - Algorithm 2 appends before it attends, so the new token attends to itself: a sequence
 *     whose cache held s rows before the step attends over n = s + 1 rows.
 *   - A sequence with n = 0 rows has no softmax; its output is defined here as zeros.
 *   - An append into a full cache (s >= L_max) is refused: the row is skipped, the length is
 *     left alone and bit 1 of *status is set.  A length outside [0, L_max] at decode time
 *     sets bit 2 and that sequence's output is zeros.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_APPEND_OVERFLOW 1
#define ORACLE_SEQLEN_RANGE 2

/* Algorithm 2, lines that write the new K/V row: K_cache[t, g, :] = k_g_new (and V alike),
 * for every key/value head g of every sequence b, at t = the sequence's current length;
 * the length then grows by one. */
void oracle_kv_append(const double *k_new, const double *v_new, double *k_cache, double *v_cache,
                      int32_t *seq_lens, int B, int H_kv, int d, int L_max, int32_t *status) {
    for (int b = 0; b < B; ++b) {
        int32_t t = seq_lens[b];
        if (t < 0 || t >= L_max) {
            if (status) *status |= ORACLE_APPEND_OVERFLOW;
            continue;
        }
        for (int g = 0; g < H_kv; ++g) {
            for (int i = 0; i < d; ++i) {
                size_t src = ((size_t)b * H_kv + g) * d + i;
                size_t dst = (((size_t)b * L_max + t) * H_kv + g) * d + i;
                k_cache[dst] = k_new[src];
                v_cache[dst] = v_new[src];
            }
        }
        seq_lens[b] = t + 1;
    }
}

/* "Expand then attend", first half: for one sequence, repeat key/value head floor(h / r)
 * for query head h.  cache_b is [L_max][H_kv][d]; out is [n][H_q][d]. */
void oracle_expand_kv(const double *cache_b, int n, int H_q, int H_kv, int d, double *out) {
    int r = H_q / H_kv;
    for (int t = 0; t < n; ++t) {
        for (int h = 0; h < H_q; ++h) {
            int g = h / r;
            for (int i = 0; i < d; ++i) {
                out[((size_t)t * H_q + h) * d + i] = cache_b[((size_t)t * H_kv + g) * d + i];
            }
        }
    }
}

/* Textbook single-head attention for one query vector, as in Algorithm 1/2 of
 * "GQA 阅读笔记": scores_t = scale * <q, K_t>, attn = softmax(scores), out = sum_t attn_t V_t.
 * K and V rows are `row_stride` doubles apart.  The softmax subtracts the largest score before
 * exponentiating (an exact identity that keeps exp() finite).  `weights` receives the n
 * softmax weights when it is not NULL. */
void oracle_attend_one_head(const double *q, const double *K, const double *V, int n, int d,
                            size_t row_stride, double scale, double *out, double *weights) {
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (n <= 0) return;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += q[i] * K[(size_t)t * row_stride + i];
        s[t] = scale * acc;
        if (s[t] > m) m = s[t];
    }
    double z = 0.0;
    for (int t = 0; t < n; ++t) {
        s[t] = exp(s[t] - m);
        z += s[t];
    }
    for (int t = 0; t < n; ++t) {
        double w = s[t] / z;
        if (weights) weights[t] = w;
        for (int i = 0; i < d; ++i) out[i] += w * V[(size_t)t * row_stride + i];
    }
    free(s);
}

/* One decode step's attention for every sequence and query head, optionally restricted to a
 * sliding window.
 *   q       [B][H_q][d]
 *   k_cache [B][L_max][H_kv][d], v_cache alike
 *   seq_lens[B]: rows each sequence attends over (already counting this step's appended row)
 *   window  > 0: every query head of sequence b attends only the last `window` rows,
 *           [max(0, n - window), n) ("GQA 阅读笔记", section on what came after GQA, Mistral
 *           7B paragraph: each token attends only the previous W tokens); <= 0: all n rows
 *   out     [B][H_q][d]
 * Per sequence: expand the attended rows (re-based so the window's first row is row 0), then
 * run textbook attention per query head.
 * Returns 0, or -1 when H_q is not a multiple of H_kv (the lesson page "r-tf2-gqa" requires
 * h to be divisible by g) or a size is not positive.  nthreads <= 0 uses the OpenMP default. */
int oracle_gqa_decode_window(const double *q, const double *k_cache, const double *v_cache,
                             const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                             int window, double scale, double *out, int nthreads,
                             int32_t *status) {
    if (B < 0 || H_q <= 0 || H_kv <= 0 || d <= 0 || L_max < 0 || H_q % H_kv != 0) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    for (int b = 0; b < B; ++b) {
        int n = seq_lens[b];
        if (n < 0 || n > L_max) {
            if (status) *status |= ORACLE_SEQLEN_RANGE;
            n = 0;
        }
        int first = (window > 0 && n > window) ? n - window : 0;
        int span = n - first;
        size_t per_seq = (size_t)L_max * H_kv * d;
        size_t row0 = (size_t)first * H_kv * d;
        size_t expanded = (size_t)span * H_q * d;
        double *Kx = (double *)malloc(sizeof(double) * (expanded ? expanded : 1));
        double *Vx = (double *)malloc(sizeof(double) * (expanded ? expanded : 1));
        oracle_expand_kv(k_cache + (size_t)b * per_seq + row0, span, H_q, H_kv, d, Kx);
        oracle_expand_kv(v_cache + (size_t)b * per_seq + row0, span, H_q, H_kv, d, Vx);
#pragma omp parallel for schedule(static)
        for (int h = 0; h < H_q; ++h) {
            oracle_attend_one_head(q + ((size_t)b * H_q + h) * d, Kx + (size_t)h * d,
                                   Vx + (size_t)h * d, span, d, (size_t)H_q * d, scale,
                                   out + ((size_t)b * H_q + h) * d, NULL);
        }
        free(Kx);
        free(Vx);
    }
    return 0;
}

/* The full decode step (no window). */
int oracle_gqa_decode(const double *q, const double *k_cache, const double *v_cache,
                      const int32_t *seq_lens, int B, int H_q, int H_kv, int d, int L_max,
                      double scale, double *out, int nthreads, int32_t *status) {
    return oracle_gqa_decode_window(q, k_cache, v_cache, seq_lens, B, H_q, H_kv, d, L_max, 0,
                                    scale, out, nthreads, status);
}

/* Several query tokens per sequence in one step (speculative decoding: "GQA 阅读笔记", what came
 * after GQA and the engineering notes -- the target model checks k drafted tokens in one pass,
 * all k queries attend the cache, which is read once).  The Q new tokens are the last Q rows
 * of the cache, and query j (0 <= j < Q) attends rows [0, n - Q + 1 + j): the prefix plus the
 * drafted tokens up to and including its own (causal among the drafts).
 *   q   [B][Q][H_q][d], caches as oracle_gqa_decode, seq_lens[b] = n (>= Q), out [B][Q][H_q][d]
 * A sequence with n < Q, n < 0 or n > L_max gets zeros and sets bit 2 of *status. */
int oracle_gqa_decode_multi(const double *q, const double *k_cache, const double *v_cache,
                            const int32_t *seq_lens, int B, int Q, int H_q, int H_kv, int d,
                            int L_max, double scale, double *out, int nthreads, int32_t *status) {
    if (B < 0 || Q <= 0 || H_q <= 0 || H_kv <= 0 || d <= 0 || L_max < 0 || H_q % H_kv != 0)
        return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    for (int b = 0; b < B; ++b) {
        int n = seq_lens[b];
        if (n < Q || n > L_max) {
            if (status) *status |= ORACLE_SEQLEN_RANGE;
            for (size_t i = 0; i < (size_t)Q * H_q * d; ++i) out[(size_t)b * Q * H_q * d + i] = 0.0;
            continue;
        }
        size_t per_seq = (size_t)L_max * H_kv * d;
        size_t expanded = (size_t)n * H_q * d;
        double *Kx = (double *)malloc(sizeof(double) * expanded);
        double *Vx = (double *)malloc(sizeof(double) * expanded);
        oracle_expand_kv(k_cache + (size_t)b * per_seq, n, H_q, H_kv, d, Kx);
        oracle_expand_kv(v_cache + (size_t)b * per_seq, n, H_q, H_kv, d, Vx);
        for (int j = 0; j < Q; ++j) {
            int rows = n - Q + 1 + j;
#pragma omp parallel for schedule(static)
            for (int h = 0; h < H_q; ++h) {
                size_t qi = (((size_t)b * Q + j) * H_q + h) * d;
                oracle_attend_one_head(q + qi, Kx + (size_t)h * d, Vx + (size_t)h * d, rows, d,
                                       (size_t)H_q * d, scale, out + qi, NULL);
            }
        }
        free(Kx);
        free(Vx);
    }
    return 0;
}

/* Paged KV cache ("GQA 阅读笔记", what came after GQA, the vLLM PagedAttention paragraph: the
 * cache is managed in fixed-size blocks; "GQA 深入理解", section 8: PagedAttention organises
 * the cache to cut fragmentation).  The cache of all sequences is one pool of pages
 *   pool [n_pages][page_size][H_kv][d]
 * and block_table[b][j] names the page that holds rows [j*page_size, (j+1)*page_size) of
 * sequence b.  Row t of sequence b is pool[block_table[b][t / page_size]][t % page_size].
 *
 * oracle_paged_gather writes the logical cache [B][max_pages*page_size][H_kv][d] of every
 * sequence (rows >= seq_lens[b] are left untouched); the paged decode is oracle_gqa_decode on
 * that gathered cache.  A page index outside [0, n_pages) for a row below seq_lens[b] sets
 * bit 4 of *status and that row is left untouched. */
void oracle_paged_gather(const double *pool, const int32_t *block_table, const int32_t *seq_lens,
                         int B, int max_pages, int page_size, int n_pages, int H_kv, int d,
                         double *cache, int32_t *status) {
    size_t L = (size_t)max_pages * page_size;
    size_t row = (size_t)H_kv * d;
    for (int b = 0; b < B; ++b) {
        int n = seq_lens[b];
        if (n < 0 || (size_t)n > L) n = 0;
        for (int t = 0; t < n; ++t) {
            int page = block_table[(size_t)b * max_pages + t / page_size];
            if (page < 0 || page >= n_pages) {
                if (status) *status |= 4;
                continue;
            }
            const double *src = pool + ((size_t)page * page_size + t % page_size) * row;
            double *dst = cache + ((size_t)b * L + t) * row;
            for (size_t i = 0; i < row; ++i) dst[i] = src[i];
        }
    }
}

/* The append of a paged cache: row t = seq_lens[b] goes to page block_table[b][t / page_size]
 * at row t % page_size; the length grows by one.  A full sequence (t >= max_pages*page_size)
 * or a page index outside [0, n_pages) is refused with bit 1 of *status. */
void oracle_kv_append_paged(const double *k_new, const double *v_new, double *k_pool,
                            double *v_pool, const int32_t *block_table, int32_t *seq_lens, int B,
                            int max_pages, int page_size, int n_pages, int H_kv, int d,
                            int32_t *status) {
    size_t row = (size_t)H_kv * d;
    for (int b = 0; b < B; ++b) {
        int t = seq_lens[b];
        if (t < 0 || t >= max_pages * page_size) {
            if (status) *status |= ORACLE_APPEND_OVERFLOW;
            continue;
        }
        int page = block_table[(size_t)b * max_pages + t / page_size];
        if (page < 0 || page >= n_pages) {
            if (status) *status |= ORACLE_APPEND_OVERFLOW;
            continue;
        }
        size_t dst = ((size_t)page * page_size + t % page_size) * row;
        for (size_t i = 0; i < row; ++i) {
            k_pool[dst + i] = k_new[(size_t)b * row + i];
            v_pool[dst + i] = v_new[(size_t)b * row + i];
        }
        seq_lens[b] = t + 1;
    }
}

/* ---------------------------------------------------------------------- FP8 (e4m3) cache
 * "GQA 阅读笔记", section "复现性与工程实践", item "混合精度": serving systems keep the KV cache
 * in FP8, and that halves the per-step KV bytes again on top of GQA's saving.  Page 3 (the
 * FlashAttention-2 GQA article), section 4.2 item 3: the cache may be stored in FP8 and
 * dequantised when read.  Neither page fixes the format or the scaling.  Reading taken here:
 * the OCP FP8 E4M3 format (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; exponent 1111 with mantissa 111 is NaN; largest finite magnitude 448), one
 * float32 scale per key/value head for K and another for V, and a stored code c of head g
 * standing for value(c) * scale[g].  Quantising x takes the code nearest to the float32
 * quotient x / scale[g] (float32 division), ties to the code with an even mantissa, and
 * magnitudes past 448 to +-448 (saturation); NaN becomes 0x7F.
 *
 * Appends and page gathers of codes reuse the float64 routines above: a code 0..255 held in a
 * double moves through them unchanged. */

/* The value a code stands for, from the field definitions. */
double oracle_e4m3_value(int code) {
    int sign = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* The code nearest to x among the finite ones, by brute force over all 127 non-negative finite
 * codes: the smallest distance wins, a tie goes to the code with an even mantissa (its lowest
 * bit clear).  Past 448 the nearest finite code is 448 itself, which is the saturation. */
int oracle_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    double a = fabs((double)x);
    /* every finite code is at most 448, so from 448 up the nearest one is 448 itself (the
     * distances of a huge x would also round to equal values) */
    if (a >= 448.0) return signbit(x) ? 0xFE : 0x7E;
    int best = 0;
    double best_dist = INFINITY;
    for (int c = 0; c < 127; ++c) {
        double dist = fabs(oracle_e4m3_value(c) - a);
        if (dist < best_dist || (dist == best_dist && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_dist = dist;
        }
    }
    return signbit(x) ? (best | 0x80) : best;
}

void oracle_e4m3_values(const uint8_t *codes, size_t n, double *out) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e4m3_value(codes[i]);
}

void oracle_e4m3_encode_array(const float *x, size_t n, uint8_t *codes) {
    for (size_t i = 0; i < n; ++i) codes[i] = (uint8_t)oracle_e4m3_encode(x[i]);
}

/* Rows of [n_rows][H_kv][d] values (each exactly a float32) to codes with per-head scales. */
void oracle_quantize_rows(const double *x, size_t n_rows, int H_kv, int d, const float *scale,
                          uint8_t *codes) {
    for (size_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < d; ++i) {
                size_t at = (r * H_kv + g) * d + i;
                float quotient = (float)x[at] / scale[g];
                codes[at] = (uint8_t)oracle_e4m3_encode(quotient);
            }
}

/* Codes of [n_rows][H_kv][d] back to values: value(code) * scale[g], exact in float64. */
void oracle_dequantize_rows(const uint8_t *codes, size_t n_rows, int H_kv, int d,
                            const float *scale, double *out) {
    for (size_t r = 0; r < n_rows; ++r)
        for (int g = 0; g < H_kv; ++g)
            for (int i = 0; i < d; ++i) {
                size_t at = (r * H_kv + g) * d + i;
                out[at] = oracle_e4m3_value(codes[at]) * (double)scale[g];
            }
}

/* Number of threads the OpenMP runtime will use for the next parallel region. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
