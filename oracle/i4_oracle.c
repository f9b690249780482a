/*
 * CPU oracle for the batch-1 INT4 weight-only decode path -- TEST INFRASTRUCTURE.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use this
 * file. It shares no code, header, table or constant with the CUDA library and
 * never calls it. Everything is computed in float64 from the plain
 * definitions; fp16 tensors are passed as raw IEEE binary16 bit patterns and
 * widened exactly.
 *
 * Source: "How To Build Your Own LLM Runtime From Scratch" (three summary
 * pages of one post). "Technical Details" names the pieces this file
 * restates: INT4 weight packing and dequantisation, a paged KV cache and
 * attention over it, with the softmax that must stay correct at page tails.
 * The pages do not print the formats; the readings used here are:
 *   - a packed word holds 8 consecutive k, field i in bits 4i..4i+3, each a
 *     two's-complement 4-bit integer in [-8, 7];
 *   - one fp16 scale per row per group of `group` consecutive k, symmetric
 *     (no zero point): W[n][k] = q[n][k] * s[n][k / group];
 *   - KV pools are [page][kv head][slot][d]; token t of a sequence lives in
 *     page page_table[t / page_size], slot t % page_size;
 *   - grouped-query attention: query head h reads kv head h / (n_q / n_kv).
 *
 * Rows are independent, so the outer loops over rows (and heads) may run on
 * several OpenMP threads; each output element is still summed by one thread
 * in increasing k (or t) order, so results do not depend on the thread count.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double half_bits_to_double(uint16_t h) {
    _Float16 f;
    memcpy(&f, &h, sizeof f);
    return (double)f;
}

static uint16_t double_to_half_bits(double d) {
    _Float16 f = (_Float16)d; /* round to nearest even, directly from double */
    uint16_t h;
    memcpy(&h, &f, sizeof h);
    return h;
}

/* Widen n fp16 values; round n float64 values to fp16 (test helpers). */
void o_f16_to_f64(const uint16_t *in, int64_t n, double *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = half_bits_to_double(in[i]);
}

void o_f64_to_f16(const double *in, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_half_bits(in[i]);
}

/* OpenMP threads of the row and head loops (n > 0 sets it); returns the count in effect. Results do not
 * depend on it: each output element is still summed by one thread in a fixed order. */
int o_set_threads(int n) {
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
}

/* Field i (0..7) of a packed word as a signed integer in [-8, 7]. */
static int int4_field(uint32_t word, int i) {
    int u = (int)((word >> (4 * i)) & 0xFu);
    return u >= 8 ? u - 16 : u;
}

/* q[n][k] = field k%8 of word w[n][k/8]. */
void o_unpack_int4(const uint32_t *w, int64_t n_rows, int64_t k_len, int8_t *q) {
    const int64_t words = k_len / 8;
    for (int64_t n = 0; n < n_rows; ++n)
        for (int64_t k = 0; k < k_len; ++k)
            q[n * k_len + k] = (int8_t)int4_field(w[n * words + k / 8], (int)(k % 8));
}

/*
 * y[m][n] = sum_k W[n][k] * x[m][k]  (+ bias[n]),  W[n][k] = q[n][k] * s[n][k/group].
 *
 * The sum runs over k = 0..K-1 in order, in float64, and the bias is added
 * last. The product q*s*x has at most 4+11+11 significant bits, so every term
 * is exact and only the running sum rounds. Four m are accumulated side by
 * side for speed; each keeps its own k order.
 */
void o_int4_linear(const uint32_t *w, const uint16_t *s, const uint16_t *x, const uint16_t *bias,
                   int64_t m_rows, int64_t n_rows, int64_t k_len, int64_t group, double *y) {
    const int64_t words = k_len / 8, groups = k_len / group;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(m_rows * k_len));
    o_f16_to_f64(x, m_rows * k_len, xd);
#pragma omp parallel
    {
        double *wrow = (double *)malloc(sizeof(double) * (size_t)k_len);
#pragma omp for schedule(static)
        for (int64_t n = 0; n < n_rows; ++n) {
            for (int64_t gi = 0; gi < groups; ++gi) {
                const double scale = half_bits_to_double(s[n * groups + gi]);
                for (int64_t k = gi * group; k < (gi + 1) * group; ++k)
                    wrow[k] = (double)int4_field(w[n * words + k / 8], (int)(k % 8)) * scale;
            }
            const double b = bias ? half_bits_to_double(bias[n]) : 0.0;
            int64_t m = 0;
            for (; m + 4 <= m_rows; m += 4) {
                const double *x0 = xd + m * k_len, *x1 = x0 + k_len, *x2 = x1 + k_len, *x3 = x2 + k_len;
                double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
                for (int64_t k = 0; k < k_len; ++k) {
                    a0 += wrow[k] * x0[k];
                    a1 += wrow[k] * x1[k];
                    a2 += wrow[k] * x2[k];
                    a3 += wrow[k] * x3[k];
                }
                y[(m + 0) * n_rows + n] = bias ? a0 + b : a0;
                y[(m + 1) * n_rows + n] = bias ? a1 + b : a1;
                y[(m + 2) * n_rows + n] = bias ? a2 + b : a2;
                y[(m + 3) * n_rows + n] = bias ? a3 + b : a3;
            }
            for (; m < m_rows; ++m) {
                const double *x0 = xd + m * k_len;
                double a0 = 0.0;
                for (int64_t k = 0; k < k_len; ++k) a0 += wrow[k] * x0[k];
                y[m * n_rows + n] = bias ? a0 + b : a0;
            }
        }
        free(wrow);
    }
    free(xd);
}

/*
 * Softmax attention of one query head over `ctx` keys given by row pointers.
 *   s_t = scale * (q . k_t),  p_t = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u),
 *   o   = sum_t p_t v_t.
 * All in float64; probabilities are returned when `probs` is not NULL.
 */
static void attend_one_head(const uint16_t *q, const uint16_t *const *krow, const uint16_t *const *vrow,
                            int64_t ctx, int64_t d, double scale, double *score, double *out, double *probs) {
    double mx = -INFINITY;
    for (int64_t t = 0; t < ctx; ++t) {
        double acc = 0.0;
        for (int64_t i = 0; i < d; ++i) acc += half_bits_to_double(q[i]) * half_bits_to_double(krow[t][i]);
        score[t] = acc * scale;
        if (score[t] > mx) mx = score[t];
    }
    double denom = 0.0;
    for (int64_t t = 0; t < ctx; ++t) {
        score[t] = exp(score[t] - mx);
        denom += score[t];
    }
    for (int64_t t = 0; t < ctx; ++t) score[t] /= denom;
    for (int64_t i = 0; i < d; ++i) out[i] = 0.0;
    for (int64_t t = 0; t < ctx; ++t)
        for (int64_t i = 0; i < d; ++i) out[i] += score[t] * half_bits_to_double(vrow[t][i]);
    if (probs)
        for (int64_t t = 0; t < ctx; ++t) probs[t] = score[t];
}

static void attend_rows(const uint16_t *q, const uint16_t *const *krows, const uint16_t *const *vrows,
                        int64_t ctx, int64_t n_q, int64_t n_kv, int64_t d, double scale, double *out,
                        double *probs) {
    const int64_t per_kv = n_q / n_kv;
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < n_q; ++h) {
        const int64_t g = h / per_kv;
        double *score = (double *)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1));
        attend_one_head(q + h * d, krows + g * ctx, vrows + g * ctx, ctx, d, scale, score, out + h * d,
                        probs ? probs + h * ctx : NULL);
        free(score);
    }
}

/*
 * Paged grouped-query decode attention for one sequence.
 * q [n_q][d]; pools [num_pages][n_kv][page_size][d]; page_table [ceil(ctx/page_size)].
 * out [n_q][d] float64; probs [n_q][ctx] (optional).
 */
void o_paged_attention(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                       const int32_t *page_table, int64_t ctx, int64_t n_q, int64_t n_kv, int64_t d,
                       int64_t page_size, double scale, double *out, double *probs) {
    const uint16_t **krows = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_kv * ctx + 1));
    const uint16_t **vrows = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_kv * ctx + 1));
    for (int64_t g = 0; g < n_kv; ++g)
        for (int64_t t = 0; t < ctx; ++t) {
            const int64_t page = page_table[t / page_size], slot = t % page_size;
            const int64_t off = ((page * n_kv + g) * page_size + slot) * d;
            krows[g * ctx + t] = k_pool + off;
            vrows[g * ctx + t] = v_pool + off;
        }
    attend_rows(q, krows, vrows, ctx, n_q, n_kv, d, scale, out, probs);
    free(krows);
    free(vrows);
}

/* The same attention over contiguous K, V [n_kv][ctx][d]. */
void o_contiguous_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t ctx, int64_t n_q,
                            int64_t n_kv, int64_t d, double scale, double *out, double *probs) {
    const uint16_t **krows = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_kv * ctx + 1));
    const uint16_t **vrows = (const uint16_t **)malloc(sizeof(void *) * (size_t)(n_kv * ctx + 1));
    for (int64_t g = 0; g < n_kv; ++g)
        for (int64_t t = 0; t < ctx; ++t) {
            krows[g * ctx + t] = k + (g * ctx + t) * d;
            vrows[g * ctx + t] = v + (g * ctx + t) * d;
        }
    attend_rows(q, krows, vrows, ctx, n_q, n_kv, d, scale, out, probs);
    free(krows);
    free(vrows);
}

/* out [n_kv][ctx][d]: the rows of one sequence's pool, in token order. */
void o_paged_gather(const uint16_t *pool, const int32_t *page_table, int64_t ctx, int64_t n_kv, int64_t d,
                    int64_t page_size, uint16_t *out) {
    for (int64_t g = 0; g < n_kv; ++g)
        for (int64_t t = 0; t < ctx; ++t) {
            const int64_t page = page_table[t / page_size], slot = t % page_size;
            memcpy(out + (g * ctx + t) * d, pool + ((page * n_kv + g) * page_size + slot) * d,
                   sizeof(uint16_t) * (size_t)d);
        }
}
