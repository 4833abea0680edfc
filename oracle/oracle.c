/*
 * oracle.c -- plain, slow, single-threaded CPU oracle of the page indexer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline / reference legs do.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only at the seeded inputs.
 *
 * What it computes, and which passage of the pages defines it
 * ------------------------------------------------------------
 * score   "Iterate Centroids Score" (opening description): the indexer scores
 *         each request's candidate pages from a batch of Q query rows and a
 *         table of block centroids.  "Round 18 Track C: qsa_topk2 ... +
 *         qsa_score Query Hoisting & Unrolling", section 1, Target 2, shows
 *         the per-page score as an FMA reduction over the query heads and the
 *         head dimension, i.e.
 *              s[b,t,p] = sum_{h<Q} sum_{d<D} q[b,t,h,d] * c[b,p,d].
 *         "Round 15 Track C Audit", section 1, Target 1 item 3, scores a tile
 *         of 16 query tokens at once (the T > 1 prefill-chunk case).
 *         Pages p >= len[b] are padding and score -inf.
 *         Inputs are bf16 bit patterns; every product of two bf16 values is
 *         exact in double, and the double sum is accumulated in h-major,
 *         d-minor order.  A[b,t,p] = sum_h sum_d |q*c| is returned beside S
 *         as the scale of the score error bound.
 * select  "Iterate Topk" (opening description): given per-segment scores,
 *         return the top-K indices.  Order: descending score; equal scores go
 *         to the lower index (IEEE equality, so -0 ties with +0: "Round 18
 *         Track C", section 2, tests signed-zero and adversarial ties).  A page
 *         is selectable iff p < len and its score is neither -inf nor NaN.
 *         K' = min(K, #selectable) entries are written, then the slots
 *         K'..K-1 get index -1 and value -inf.
 *         The selection is a full sort (C library qsort) of the selectable
 *         entries under the total order (value desc, index asc); because the
 *         order is total, the result equals a stable sort by value.
 *
 * Error behaviour: every entry point returns 0 on success and -1 when an
 * argument breaks the contract (negative sizes, len outside [0, N]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* bf16 bit pattern -> double, exactly: the bf16 value is the fp32 value whose
 * high 16 bits are the pattern and whose low 16 bits are zero. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One score and its error-bound scale, by the definition. */
static void score_one(const uint16_t* q_bt, const uint16_t* c_bp, int Q, int D,
                      double* s_out, double* a_out)
{
    double s = 0.0, a = 0.0;
    for (int h = 0; h < Q; ++h) {
        for (int d = 0; d < D; ++d) {
            double prod = bf16_bits_to_double(q_bt[(int64_t)h * D + d]) *
                          bf16_bits_to_double(c_bp[d]);
            s += prod;
            a += fabs(prod);
        }
    }
    *s_out = s;
    *a_out = a;
}

/*
 * Scores of every (b, t, p).
 *   q        bf16 bits [B][T][Q][D]
 *   c        bf16 bits, request b's page p at c + b*ldc_b + p*D  (p < N)
 *   lengths  [B] valid page counts in [0, N], or NULL for "all N valid"
 *   S, A     double [B][T][N]; padded entries get S = -inf, A = 0
 */
ORACLE_API int oracle_scores(const uint16_t* q, const uint16_t* c,
                             const int32_t* lengths, int B, int T, int Q, int D,
                             int N, int64_t ldc_b, double* S, double* A)
{
    if (B < 0 || T < 0 || Q <= 0 || D <= 0 || N < 0 || ldc_b < (int64_t)N * D)
        return -1;
    for (int b = 0; b < B; ++b) {
        int len = lengths ? lengths[b] : N;
        if (len < 0 || len > N) return -1;
        for (int t = 0; t < T; ++t) {
            const uint16_t* q_bt = q + ((int64_t)b * T + t) * Q * D;
            double* s_row = S + ((int64_t)b * T + t) * N;
            double* a_row = A + ((int64_t)b * T + t) * N;
            for (int p = 0; p < N; ++p) {
                if (p >= len) {
                    s_row[p] = -INFINITY;
                    a_row[p] = 0.0;
                    continue;
                }
                score_one(q_bt, c + (int64_t)b * ldc_b + (int64_t)p * D, Q, D,
                          &s_row[p], &a_row[p]);
            }
        }
    }
    return 0;
}

/*
 * Scores with a valid page count per (request, token): multi-token decode
 * where token t of request b sees only the pages before its own position
 * (the per-token "dead" tail of "Round 15 Track C Audit", section 1 Target 1
 * item 3, and the pos0 x ntok grid of "Round 18 Track C", section 2).
 *   tok_lengths  [B][T] valid page counts in [0, N]
 *   S, A         double [B][T][N]; entries p >= tok_lengths[b][t] get
 *                S = -inf, A = 0
 */
ORACLE_API int oracle_scores_tokens(const uint16_t* q, const uint16_t* c,
                                    const int32_t* tok_lengths, int B, int T,
                                    int Q, int D, int N, int64_t ldc_b,
                                    double* S, double* A)
{
    if (B < 0 || T < 0 || Q <= 0 || D <= 0 || N < 0 || ldc_b < (int64_t)N * D ||
        !tok_lengths)
        return -1;
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < T; ++t) {
            const int len = tok_lengths[(int64_t)b * T + t];
            if (len < 0 || len > N) return -1;
            const uint16_t* q_bt = q + ((int64_t)b * T + t) * Q * D;
            double* s_row = S + ((int64_t)b * T + t) * N;
            double* a_row = A + ((int64_t)b * T + t) * N;
            for (int p = 0; p < N; ++p) {
                if (p >= len) {
                    s_row[p] = -INFINITY;
                    a_row[p] = 0.0;
                    continue;
                }
                score_one(q_bt, c + (int64_t)b * ldc_b + (int64_t)p * D, Q, D,
                          &s_row[p], &a_row[p]);
            }
        }
    }
    return 0;
}

typedef struct {
    double v;
    int32_t i;
} entry;

/* Total order: larger value first; equal values (including -0 == +0) by
 * ascending index. */
static int entry_cmp(const void* pa, const void* pb)
{
    const entry* a = (const entry*)pa;
    const entry* b = (const entry*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

/* Core select over a row already widened to double (exact for fp32 input). */
static int topk_core(const double* row, int len, int K, int32_t* idx_out,
                     double* val_out)
{
    if (len < 0 || K < 0) return -1;
    entry* e = (entry*)malloc(sizeof(entry) * (size_t)(len > 0 ? len : 1));
    if (!e) return -1;
    int n = 0;
    for (int p = 0; p < len; ++p) {
        double v = row[p];
        if (isnan(v) || v == -INFINITY) continue;
        e[n].v = v;
        e[n].i = p;
        ++n;
    }
    qsort(e, (size_t)n, sizeof(entry), entry_cmp);
    int kk = n < K ? n : K;
    for (int k = 0; k < K; ++k) {
        idx_out[k] = k < kk ? e[k].i : -1;
        val_out[k] = k < kk ? e[k].v : -INFINITY;
    }
    free(e);
    return kk;
}

/* Top-K of one double row; returns K' (the number of real entries) or -1. */
ORACLE_API int oracle_topk_f64(const double* row, int len, int K,
                               int32_t* idx_out, double* val_out)
{
    return topk_core(row, len, K, idx_out, val_out);
}

/* Top-K of one fp32 row.  Widening fp32 to double is exact, so every
 * comparison decides exactly as the same comparison in fp32 would. */
ORACLE_API int oracle_topk_f32(const float* row, int len, int K,
                               int32_t* idx_out, float* val_out)
{
    if (len < 0 || K < 0) return -1;
    double* w = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
    double* v = (double*)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1));
    if (!w || !v) {
        free(w);
        free(v);
        return -1;
    }
    for (int p = 0; p < len; ++p) w[p] = (double)row[p];
    int kk = topk_core(w, len, K, idx_out, v);
    /* The value written is the row's own fp32 entry (bit-exact, -0 kept). */
    for (int k = 0; k < K; ++k) val_out[k] = idx_out[k] >= 0 ? row[idx_out[k]] : -INFINITY;
    free(w);
    free(v);
    return kk;
}

/* Row-batched fp32 select: rows of stride lds, lengths per row (NULL => N). */
ORACLE_API int oracle_topk_rows_f32(const float* scores, const int32_t* lengths,
                                    int rows, int N, int64_t lds, int K,
                                    int32_t* idx_out, float* val_out)
{
    if (rows < 0 || N < 0 || K < 0 || lds < N) return -1;
    for (int r = 0; r < rows; ++r) {
        int len = lengths ? lengths[r] : N;
        if (len < 0 || len > N) return -1;
        if (oracle_topk_f32(scores + (int64_t)r * lds, len, K,
                            idx_out + (int64_t)r * K, val_out + (int64_t)r * K) < 0)
            return -1;
    }
    return 0;
}

/* Row-batched double select (the oracle's own scores). */
ORACLE_API int oracle_topk_rows_f64(const double* scores, const int32_t* lengths,
                                    int rows, int N, int64_t lds, int K,
                                    int32_t* idx_out, double* val_out)
{
    if (rows < 0 || N < 0 || K < 0 || lds < N) return -1;
    for (int r = 0; r < rows; ++r) {
        int len = lengths ? lengths[r] : N;
        if (len < 0 || len > N) return -1;
        if (topk_core(scores + (int64_t)r * lds, len, K, idx_out + (int64_t)r * K,
                      val_out + (int64_t)r * K) < 0)
            return -1;
    }
    return 0;
}

/*
 * Page centroids by key mean-pooling (the "pooled keys" that feed the
 * indexer, "Round 15 Track C Audit", section 2 parity list): request b holds
 * key_counts[b] keys of D bf16 values at keys + b*ldk_b + i*D; page p covers
 * keys p*P .. p*P + P - 1, and its centroid is the mean of the page's valid
 * keys, n = min(P, key_counts[b] - p*P), computed exactly in double.
 *   means  double [B][N][D]; pages with no valid key get 0
 * Returns -1 on arguments outside the contract.
 */
ORACLE_API int oracle_pool(const uint16_t* keys, const int32_t* key_counts, int B, int D, int P,
                           int N, int64_t ldk_b, double* means)
{
    if (B < 0 || D <= 0 || P <= 0 || N < 0 || !key_counts) return -1;
    for (int b = 0; b < B; ++b) {
        const int nk = key_counts[b];
        if (nk < 0 || (int64_t)nk > (int64_t)N * P || ldk_b < (int64_t)nk * D) return -1;
        for (int p = 0; p < N; ++p) {
            double* m = means + ((int64_t)b * N + p) * D;
            int n = nk - p * P;
            n = n < 0 ? 0 : (n > P ? P : n);
            for (int d = 0; d < D; ++d) {
                double s = 0.0;
                for (int i = 0; i < n; ++i)
                    s += bf16_bits_to_double(keys[(int64_t)b * ldk_b + ((int64_t)p * P + i) * D + d]);
                m[d] = n ? s / n : 0.0;
            }
        }
    }
    return 0;
}

/*
 * KMeans assignment ("Export Cake KMeans plan-runtime suite", summary:
 * assignments = runtime.compute(x, centroids) on raw bf16 inputs): every
 * point goes to its nearest centroid in Euclidean distance.  Since
 * |x - c|^2 = |x|^2 - 2 (x.c - |c|^2 / 2) and |x|^2 does not depend on c,
 * the nearest centroid is the one of largest
 *     s[i,c] = sum_d x[i,d] * c[c,d] - (sum_d c[c,d]^2) / 2,
 * computed here in double (bf16 products and squares are exact in double).
 * Equal scores go to the lower centroid index.
 *   x       bf16 bits [M][D], centroids bf16 bits [C][D]
 *   assign  int32 [M]; best double [M] (the winning score)
 *   S, A    optional (NULL) double [M][C]: every score, and the scale of its
 *           error bound, sum_d |x*c| + (sum_d c^2) / 2
 * Returns -1 on arguments outside the contract.
 */
ORACLE_API int oracle_kmeans_assign(const uint16_t* x, const uint16_t* cent, int M, int C, int D,
                                    int32_t* assign, double* best, double* S, double* A)
{
    if (M < 0 || C <= 0 || D <= 0 || !assign || !best) return -1;
    for (int i = 0; i < M; ++i) {
        int arg = 0;
        double top = 0.0;
        for (int c = 0; c < C; ++c) {
            double dot = 0.0, mag = 0.0, half = 0.0;
            for (int d = 0; d < D; ++d) {
                const double xv = bf16_bits_to_double(x[(int64_t)i * D + d]);
                const double cv = bf16_bits_to_double(cent[(int64_t)c * D + d]);
                dot += xv * cv;
                mag += fabs(xv * cv);
                half += cv * cv;
            }
            half *= 0.5;
            const double s = dot - half;
            if (S) S[(int64_t)i * C + c] = s;
            if (A) A[(int64_t)i * C + c] = mag + half;
            if (c == 0 || s > top) {  /* strictly greater: ties keep the lower index */
                top = s;
                arg = c;
            }
        }
        assign[i] = arg;
        best[i] = top;
    }
    return 0;
}

/*
 * Argmax of every row of an fp32 score matrix [M][C] (ties to the lower
 * column; NaN never wins, a row of NaN gives -1), for the bit-exact check of
 * an assignment against the GPU's own scores.
 */
ORACLE_API int oracle_argmax_rows_f32(const float* S, int M, int C, int32_t* arg)
{
    if (M < 0 || C <= 0 || !arg) return -1;
    for (int i = 0; i < M; ++i) {
        int a = -1;
        float top = 0.0f;
        for (int c = 0; c < C; ++c) {
            const float v = S[(int64_t)i * C + c];
            if (v != v) continue;
            if (a < 0 || v > top) {
                top = v;
                a = c;
            }
        }
        arg[i] = a;
    }
    return 0;
}
