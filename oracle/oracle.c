/*
 * oracle.c -- plain, slow CPU reference for two-stage bucketed approximate top-k.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this code.  It shares nothing with the
 * CUDA library: no headers, no helpers, no tables.
 *
 * Source: "Approximate Top-k for Increased Parallelism" (Key, Ribar, Cattaneo,
 * Hudlass-Galley, Orr; arXiv 2412.04358), as summarised on its pith.science
 * review page:
 *   - "What carries the argument": the n inputs are split into b interleaved
 *     buckets, an exact top-k_b is taken inside every bucket, and when the
 *     b*k_b concatenated candidates exceed k a final exact top-k keeps the k
 *     largest.
 *   - Fig. 2 (n=11, k=4, b=3, k_b=2): Stage 1 reduces n elements to b*k_b
 *     candidates, Stage 2 takes the final top-k.
 *   - "The reading": element i belongs to bucket i mod b (interleaved).
 * The fused scoring step (score = q . K_i over a key cache) follows the
 * selector described on "Recall Before You Rank" (ReTopK, abstract: the
 * current query is scored against the full KV cache before a global top-K)
 * and the STARC page, Fig. 3 (q in R^{1 x d_h}, K in R^{L x d_h}).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - Ties: equal values rank by lowest index.  IEEE equality is used, so
 *     -0.0 and +0.0 tie.  NaN ranks above +inf; all NaNs are equal.
 *   - When b does not divide n, bucket j holds the indices i < n with
 *     i mod b == j (so sizes differ by at most one; empty when j >= n).
 *   - Output: the kept elements sorted best-first; slots past the number of
 *     candidates hold value -inf and index -1.  Values are the input bits.
 *   - Scores: bf16 x bf16 products are exact in double; the sum is taken in
 *     double in index order of d and rounded once to float.  No 1/sqrt(d).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    float v;
    int64_t i;
} item;

/* a ranks strictly before b under the total order (value desc, index asc). */
static int ranks_before(const item *a, const item *b)
{
    int an = isnan(a->v), bn = isnan(b->v);
    if (an || bn) {
        if (an && bn)
            return a->i < b->i;
        return an; /* NaN is above every number */
    }
    if (a->v > b->v)
        return 1;
    if (a->v < b->v)
        return 0;
    return a->i < b->i; /* equal values (incl. -0 == +0): lower index first */
}

static int cmp_items(const void *x, const void *y)
{
    const item *a = (const item *)x, *b = (const item *)y;
    if (ranks_before(a, b))
        return -1;
    if (ranks_before(b, a))
        return 1;
    return 0;
}

static void write_row(const item *sorted, int64_t keep, int64_t k, float *ov, int32_t *oi)
{
    for (int64_t s = 0; s < k; ++s) {
        if (s < keep) {
            ov[s] = sorted[s].v;
            oi[s] = (int32_t)sorted[s].i;
        } else {
            ov[s] = -INFINITY;
            oi[s] = -1;
        }
    }
}

/* Stage 1 + Stage 2 for one row of n values. Returns the candidate count C. */
static int64_t bucketed_row(const float *x, int64_t n, int64_t k, int64_t b, int64_t kb,
                            float *ov, int32_t *oi, item *bucket, item *cand)
{
    int64_t C = 0;
    /* Stage 1: every interleaved bucket j = {i : i mod b == j} keeps its exact top-k_b. */
    for (int64_t j = 0; j < b; ++j) {
        int64_t m = 0;
        for (int64_t i = j; i < n; i += b) {
            bucket[m].v = x[i];
            bucket[m].i = i;
            ++m;
        }
        qsort(bucket, (size_t)m, sizeof(item), cmp_items);
        int64_t take = m < kb ? m : kb;
        for (int64_t t = 0; t < take; ++t)
            cand[C++] = bucket[t];
    }
    /* Stage 2: if the candidates exceed k, keep the k best; the kept ones are
     * returned best-first either way. */
    qsort(cand, (size_t)C, sizeof(item), cmp_items);
    int64_t keep = C < k ? C : k;
    write_row(cand, keep, k, ov, oi);
    return C;
}

static int g_threads = 1;

void oracle_set_threads(int t) { g_threads = t > 0 ? t : 1; }

int oracle_get_threads(void) { return g_threads; }

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_num_procs();
#else
    return 1;
#endif
}

/* Bucketed approximate top-k over `rows` rows of n floats (row-major).
 * out_vals/out_idx: rows*k.  out_cand (nullable): per-row candidate count C. */
int oracle_bucketed(const float *x, int64_t rows, int64_t n, int64_t k, int64_t b, int64_t kb,
                    float *out_vals, int32_t *out_idx, int64_t *out_cand)
{
    if (rows < 0 || n < 1 || k < 1 || b < 1 || kb < 1)
        return 1;
    int64_t bmax = (n + b - 1) / b;
    int64_t cmax = b * kb < n ? b * kb : n;
    int fail = 0;
#pragma omp parallel num_threads(g_threads)
    {
        item *bucket = (item *)malloc(sizeof(item) * (size_t)(bmax > 0 ? bmax : 1));
        item *cand = (item *)malloc(sizeof(item) * (size_t)(cmax > 0 ? cmax : 1));
        if (!bucket || !cand) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < rows; ++r) {
                int64_t C = bucketed_row(x + r * n, n, k, b, kb, out_vals + r * k,
                                         out_idx + r * k, bucket, cand);
                if (out_cand)
                    out_cand[r] = C;
            }
        }
        free(bucket);
        free(cand);
    }
    return fail ? 2 : 0;
}

/* Exact top-k: the first min(k, n) elements of each row under the total order. */
int oracle_exact(const float *x, int64_t rows, int64_t n, int64_t k, float *out_vals,
                 int32_t *out_idx)
{
    if (rows < 0 || n < 1 || k < 1)
        return 1;
    int fail = 0;
#pragma omp parallel num_threads(g_threads)
    {
        item *all = (item *)malloc(sizeof(item) * (size_t)n);
        if (!all) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < rows; ++r) {
                const float *row = x + r * n;
                for (int64_t i = 0; i < n; ++i) {
                    all[i].v = row[i];
                    all[i].i = i;
                }
                qsort(all, (size_t)n, sizeof(item), cmp_items);
                write_row(all, n < k ? n : k, k, out_vals + r * k, out_idx + r * k);
            }
        }
        free(all);
    }
    return fail ? 2 : 0;
}

/* Bucketed selection over an arbitrary candidate list of (value, index) pairs:
 * the bucket of a pair is its index mod b (not its position in the list).
 * Used to state the split-and-merge property of the method. */
int oracle_bucketed_pairs(const float *v, const int32_t *idx, int64_t m, int64_t k, int64_t b,
                          int64_t kb, float *out_vals, int32_t *out_idx)
{
    if (m < 0 || k < 1 || b < 1 || kb < 1)
        return 1;
    item *all = (item *)malloc(sizeof(item) * (size_t)(m > 0 ? m : 1));
    item *bucket = (item *)malloc(sizeof(item) * (size_t)(m > 0 ? m : 1));
    item *cand = (item *)malloc(sizeof(item) * (size_t)(m > 0 ? m : 1));
    if (!all || !bucket || !cand) {
        free(all);
        free(bucket);
        free(cand);
        return 2;
    }
    for (int64_t t = 0; t < m; ++t) {
        all[t].v = v[t];
        all[t].i = idx[t];
    }
    int64_t C = 0;
    for (int64_t j = 0; j < b; ++j) {
        int64_t cnt = 0;
        for (int64_t t = 0; t < m; ++t)
            if (all[t].i % b == j)
                bucket[cnt++] = all[t];
        qsort(bucket, (size_t)cnt, sizeof(item), cmp_items);
        int64_t take = cnt < kb ? cnt : kb;
        for (int64_t t = 0; t < take; ++t)
            cand[C++] = bucket[t];
    }
    qsort(cand, (size_t)C, sizeof(item), cmp_items);
    write_row(cand, C < k ? C : k, k, out_vals, out_idx);
    free(all);
    free(bucket);
    free(cand);
    return 0;
}

/* Sampling tail of vocabulary sampling (the review page's "Core claim":
 * top-k vocabulary sampling with n = 128,256 and k = 256 is one of the three
 * workloads; Fig. 4, left).  The pages do not write the tail out; this is the
 * plain reading of top-k sampling.  From the selected (value, index) pairs of
 * one row, best-first, index idx[i] is drawn with probability
 *     w_i / sum_j w_j,   w_i = exp((v_i - v_0) / T),
 * by inverse CDF with the caller's uniform u in [0, 1): the first i whose
 * running sum of w exceeds u * sum w (the last positive-weight entry if
 * rounding leaves none).  Padding (index -1) and -inf values weigh 0.  When
 * v_0 is NaN or +inf the draw is idx[0]; with no candidate it is -1.  All in
 * double.  *margin receives min_i |running_sum_i - u * sum| / sum, the
 * relative distance of the draw from its nearest CDF boundary. */
int oracle_sample_row(const float *v, const int32_t *idx, int64_t k, double inv_t, double u,
                      int32_t *token, double *margin)
{
    *margin = INFINITY;
    if (k < 1 || idx[0] < 0) {
        *token = -1;
        return 0;
    }
    if (isnan(v[0]) || (isinf(v[0]) && v[0] > 0)) {
        *token = idx[0];
        return 0;
    }
    double total = 0.0;
    for (int64_t i = 0; i < k; ++i)
        if (idx[i] >= 0)
            total += exp(((double)v[i] - (double)v[0]) * inv_t);
    const double target = u * total;
    double run = 0.0;
    int32_t pick = -1, last = -1;
    for (int64_t i = 0; i < k; ++i) {
        if (idx[i] < 0)
            continue;
        const double w = exp(((double)v[i] - (double)v[0]) * inv_t);
        if (w > 0.0)
            last = idx[i];
        run += w;
        const double gap = fabs(run - target) / total;
        if (gap < *margin)
            *margin = gap;
        if (pick < 0 && run > target)
            pick = idx[i];
    }
    *token = pick >= 0 ? pick : last;
    return 0;
}

static double bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* score[r][i] = sum_d q[r][d] * K[r*kstride + i*d_dim + d], accumulated in
 * double, rounded once to float.  kstride is in elements; 0 shares one K. */
int oracle_scores(const uint16_t *q, int64_t rows, int64_t d, const uint16_t *K, int64_t n,
                  int64_t kstride, float *out)
{
    if (rows < 0 || d < 1 || n < 1 || kstride < 0)
        return 1;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t *qr = q + r * d;
        const uint16_t *Kr = K + r * kstride;
        for (int64_t i = 0; i < n; ++i) {
            double s = 0.0;
            for (int64_t t = 0; t < d; ++t)
                s += bf16_to_double(qr[t]) * bf16_to_double(Kr[i * d + t]);
            out[r * n + i] = (float)s;
        }
    }
    return 0;
}

/* Re-ranking of a candidate index set ("Recall Before You Rank", abstract:
 * the supports of similar earlier queries are reused as candidates and
 * scored exactly against the current query before the top-K is kept).  Per
 * row r: the distinct indices 0 <= i < n among cand[r][0..c) (-1 marks an
 * empty slot; repeats and out-of-range indices are dropped), each scored as
 * in oracle_scores, and the k best (score, index) pairs under the total
 * order, best-first, padded with -inf / -1. */
int oracle_rerank(const uint16_t *q, int64_t rows, int64_t d, const uint16_t *K, int64_t n,
                  int64_t kstride, const int32_t *cand, int64_t c, int64_t k, float *out_vals,
                  int32_t *out_idx)
{
    if (rows < 0 || d < 1 || n < 1 || c < 1 || k < 1 || kstride < 0)
        return 1;
    int fail = 0;
#pragma omp parallel num_threads(g_threads)
    {
        item *all = (item *)malloc(sizeof(item) * (size_t)c);
        if (!all) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            if (!all)
                continue;
            const uint16_t *qr = q + r * d;
            const uint16_t *Kr = K + kstride * r; /* this row's key matrix */
            const int32_t *cr = cand + r * c;
            int64_t m = 0;
            for (int64_t j = 0; j < c; ++j) {
                const int64_t i = cr[j];
                if (i < 0 || i >= n)
                    continue;
                int seen = 0;
                for (int64_t t = 0; t < m && !seen; ++t)
                    seen = all[t].i == i;
                if (seen)
                    continue;
                double acc = 0.0; /* exact bf16 products, summed over t in order */
                for (int64_t t = 0; t < d; ++t)
                    acc += bf16_to_double(Kr[i * d + t]) * bf16_to_double(qr[t]);
                all[m].v = (float)acc;
                all[m].i = i;
                ++m;
            }
            qsort(all, (size_t)m, sizeof(item), cmp_items);
            write_row(all, m < k ? m : k, k, out_vals + r * k, out_idx + r * k);
        }
        free(all);
    }
    return fail ? 2 : 0;
}

/* Fused scoring then bucketed selection on the float scores. out_scores
 * (nullable) receives the rows*n float scores. */
int oracle_score_topk(const uint16_t *q, int64_t rows, int64_t d, const uint16_t *K, int64_t n,
                      int64_t kstride, int64_t k, int64_t b, int64_t kb, float *out_vals,
                      int32_t *out_idx, float *out_scores)
{
    if (rows < 0 || d < 1 || n < 1 || k < 1 || b < 1 || kb < 1 || kstride < 0)
        return 1;
    float *scores = out_scores;
    if (!scores) {
        scores = (float *)malloc(sizeof(float) * (size_t)(rows * n > 0 ? rows * n : 1));
        if (!scores)
            return 2;
    }
    int rc = oracle_scores(q, rows, d, K, n, kstride, scores);
    if (rc == 0)
        rc = oracle_bucketed(scores, rows, n, k, b, kb, out_vals, out_idx, NULL);
    if (!out_scores)
        free(scores);
    return rc;
}
