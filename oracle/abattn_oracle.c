/*
 * AB-Attention CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, double-precision restatement of what the AB-Attention hot path
 * computes.  Only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * Sources (the two pages about the method):
 *  [P1] "AB-Attention: Video Difuzyon Transformer'larini Hizlandirmak Icin Dogru
 *       Blok Dikkat Mekanizmasi" (edumints blog), sections "Video Difuzyon
 *       Modellerinde Dikkat Darbogazi" (bottleneck) and "AB-Attention ve Uc
 *       Temel Yenilig(i)" (three innovations).
 *  [P2] "AB-Attention yusarri' tawlid al-video hatta 2,23x ..." (hamidun news,
 *       Arabic), sections "where earlier sparse schemes fail" and "three
 *       techniques in AB-Attention" (IBCS / SIP / fine-grained kernel
 *       paragraphs).
 * Steps the pages leave open are resolved with the plainest reading; each
 * such reading is marked READING below.
 *
 * Layout: one head at a time, row-major double arrays [N][d]; the batch
 * drivers at the end take [B][H][N][d] and run rows (b, h, q-block) in
 * parallel with OpenMP.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Mean keys.  [P2] IBCS paragraph: a KV block is scored through its mean key.
 * kbar_j = (1/|j|) sum_{t in block j} k_t, where a ragged last block uses its
 * true number of keys (READING).                                            */
void oc_meanpool(const double *K, int64_t N, int64_t d, int64_t kb, double *Kbar)
{
    int64_t nkvb = (N + kb - 1) / kb;
    for (int64_t j = 0; j < nkvb; ++j) {
        int64_t t0 = j * kb, t1 = t0 + kb < N ? t0 + kb : N;
        for (int64_t c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int64_t t = t0; t < t1; ++t) acc += K[t * d + c];
            Kbar[j * d + c] = acc / (double)(t1 - t0);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Intra-block k-means.  [P2] IBCS paragraph: the queries of each 128-query
 * block are grouped into 8 clusters, each with a centroid and a weight equal
 * to its share of the block's queries; tokens are never reordered.
 * READING (the pages give no procedure): Lloyd's algorithm with squared
 * Euclidean distance; centroid c starts at query floor(c*M/nc); each
 * iteration assigns every query to its nearest centroid (ties -> lowest c) and
 * then moves each centroid to the mean of its members (an empty cluster keeps
 * its centroid); weights come from the last assignment.                     */
void oc_kmeans(const double *Qb, int64_t M, int64_t d, int nc, int iters,
               double *C, double *w, int32_t *labels)
{
    for (int c = 0; c < nc; ++c) {
        int64_t src = ((int64_t)c * M) / nc;
        memcpy(C + (int64_t)c * d, Qb + src * d, sizeof(double) * d);
    }
    double *sum = (double *)calloc((size_t)nc * d, sizeof(double));
    int64_t *cnt = (int64_t *)calloc((size_t)nc, sizeof(int64_t));
    for (int it = 0; it < iters; ++it) {
        for (int64_t i = 0; i < M; ++i) {
            int best = 0;
            double bestd = INFINITY;
            for (int c = 0; c < nc; ++c) {
                double dist = 0.0;
                for (int64_t k = 0; k < d; ++k) {
                    double diff = Qb[i * d + k] - C[(int64_t)c * d + k];
                    dist += diff * diff;
                }
                if (dist < bestd) { bestd = dist; best = c; }
            }
            labels[i] = best;
        }
        memset(sum, 0, sizeof(double) * nc * d);
        memset(cnt, 0, sizeof(int64_t) * nc);
        for (int64_t i = 0; i < M; ++i) {
            cnt[labels[i]] += 1;
            for (int64_t k = 0; k < d; ++k) sum[(int64_t)labels[i] * d + k] += Qb[i * d + k];
        }
        for (int c = 0; c < nc; ++c)
            if (cnt[c] > 0)
                for (int64_t k = 0; k < d; ++k)
                    C[(int64_t)c * d + k] = sum[(int64_t)c * d + k] / (double)cnt[c];
    }
    for (int c = 0; c < nc; ++c) w[c] = (double)cnt[c] / (double)M;
    if (iters == 0) {  /* no assignment ever made: weights undefined -> uniform */
        for (int c = 0; c < nc; ++c) w[c] = 1.0 / nc;
    }
    free(sum);
    free(cnt);
}

/* ------------------------------------------------------------------------ */
/* Block scores.  [P2] IBCS paragraph: a KV block's score is the weighted
 * attention of the centroids to its mean key, so a block seen by a single
 * cluster keeps that cluster's share.  READING: each centroid's attention is
 * the softmax over all KV blocks of scale * c . kbar_j (scale = 1/sqrt(d) by
 * default), and s_j = sum_c w_c softmax_j(...), which sums to 1.            */
void oc_scores(const double *C, const double *w, int nc, const double *Kbar,
               int64_t nkvb, int64_t d, double scale, double *s)
{
    double *L = (double *)malloc(sizeof(double) * nkvb);
    for (int64_t j = 0; j < nkvb; ++j) s[j] = 0.0;
    for (int c = 0; c < nc; ++c) {
        double m = -INFINITY;
        for (int64_t j = 0; j < nkvb; ++j) {
            double dot = 0.0;
            for (int64_t k = 0; k < d; ++k) dot += C[(int64_t)c * d + k] * Kbar[j * d + k];
            L[j] = scale * dot;
            if (L[j] > m) m = L[j];
        }
        double Z = 0.0;
        for (int64_t j = 0; j < nkvb; ++j) Z += exp(L[j] - m);
        for (int64_t j = 0; j < nkvb; ++j) s[j] += w[c] * exp(L[j] - m) / Z;
    }
    free(L);
}

/* ------------------------------------------------------------------------ */
/* Inclusion probabilities.  [P1] SIP bullet and [P2] SIP paragraph: a block's
 * inclusion probability is proportional to its score, and the most important
 * blocks are always taken.  READING: pi_j = min(1, lambda * s_j) with
 * sum_j pi_j = Bblk (the expected number of selected blocks), found by the
 * capping iteration below; blocks with s_j = 0 get pi_j = 0.  Returns the
 * number of capping rounds; *lambda_out receives lambda (0 when every
 * positive-score block is capped).                                          */
int oc_waterfill(const double *s, int64_t n, double Bblk, double *pi, double *lambda_out)
{
    int64_t npos = 0;
    for (int64_t j = 0; j < n; ++j) npos += s[j] > 0.0;
    if (Bblk >= (double)npos) {
        for (int64_t j = 0; j < n; ++j) pi[j] = s[j] > 0.0 ? 1.0 : 0.0;
        if (lambda_out) *lambda_out = 0.0;
        return 0;
    }
    unsigned char *capped = (unsigned char *)calloc((size_t)(n > 0 ? n : 1), 1);
    int64_t ncap = 0;
    double lambda = 0.0;
    int rounds = 0;
    for (;;) {
        double rest = 0.0;
        for (int64_t j = 0; j < n; ++j)
            if (!capped[j]) rest += s[j];
        lambda = (Bblk - (double)ncap) / rest;
        int64_t added = 0;
        for (int64_t j = 0; j < n; ++j)
            if (!capped[j] && lambda * s[j] >= 1.0) { capped[j] = 1; ++added; }
        ++rounds;
        if (added == 0) break;
        ncap += added;
    }
    for (int64_t j = 0; j < n; ++j) pi[j] = capped[j] ? 1.0 : lambda * s[j];
    if (lambda_out) *lambda_out = lambda;
    free(capped);
    return rounds;
}

/* ------------------------------------------------------------------------ */
/* Counter-based uniform.  The pages name no generator.  READING: Philox4x64
 * with 10 rounds (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC'11): each round multiplies words 0 and 2 by two fixed
 * odd constants, takes the 128-bit products' high and low halves, and mixes
 * the high halves with words 1 and 3 and the round key; the key is bumped by
 * two Weyl constants between rounds.                                         */
static void mul128(uint64_t a, uint64_t b, uint64_t *hi, uint64_t *lo)
{
    unsigned __int128 p = (unsigned __int128)a * (unsigned __int128)b;
    *hi = (uint64_t)(p >> 64);
    *lo = (uint64_t)p;
}

void oc_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4])
{
    const uint64_t M0 = 0xD2E7470EE14C6C93ULL, M1 = 0xCA5A826395121157ULL;
    const uint64_t W0 = 0x9E3779B97F4A7C15ULL, W1 = 0xBB67AE8584CAA73BULL;
    uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t hi0, lo0, hi1, lo1;
        mul128(M0, x0, &hi0, &lo0);
        mul128(M1, x2, &hi1, &lo1);
        uint64_t y0 = hi1 ^ x1 ^ k0, y1 = lo1, y2 = hi0 ^ x3 ^ k1, y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += W0;
        k1 += W1;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The uniform for KV block j of row (b, h, qb): counter (j / 8, qb, h, b),
 * key (seed, 0); 64-bit word (j / 2) % 4 of the block supplies two draws, its
 * high 32-bit half for even j and its low half for odd j; the top 24 bits of
 * that half give u = bits * 2^-24, exactly representable in float32
 * (READING: the pages name no generator).                                   */
float oc_uniform(uint64_t seed, int64_t b, int64_t h, int64_t qb, int64_t j)
{
    uint64_t ctr[4] = {(uint64_t)(j >> 3), (uint64_t)qb, (uint64_t)h, (uint64_t)b};
    uint64_t key[2] = {seed, 0};
    uint64_t out[4];
    oc_philox4x64_10(ctr, key, out);
    uint64_t w = out[(j >> 1) & 3];
    uint32_t half = (j & 1) ? (uint32_t)w : (uint32_t)(w >> 32);
    return (float)(half >> 8) * 0x1p-24f;
}

/* Poisson sampling.  [P2] SIP paragraph: each block enters the sample on its
 * own with its inclusion probability.  Block j is taken iff u_j < pi_j, the
 * comparison made in float32 so pi = 1 is always and pi = 0 never taken;
 * selected indices are written in ascending order (READING).  Writes at most
 * cap entries and returns the true count.                                   */
int64_t oc_sample(const float *pi, int64_t n, uint64_t seed, int64_t b, int64_t h,
                  int64_t qb, int32_t *idx, float *pi_sel, int64_t cap)
{
    int64_t cnt = 0;
    for (int64_t j = 0; j < n; ++j) {
        float u = oc_uniform(seed, b, h, qb, j);
        if (u < pi[j]) {
            if (cnt < cap) { idx[cnt] = (int32_t)j; pi_sel[cnt] = pi[j]; }
            ++cnt;
        }
    }
    return cnt;
}

/* Truncation baseline.  [P2] "where earlier sparse schemes fail", second
 * weakness: top-k keeps the k best blocks and drops the rest from both the
 * numerator and the normaliser.  k highest scores, ties -> lower index,
 * returned in ascending index order; each kept block has weight 1.          */
typedef struct { double s; int32_t j; } oc_scored;
static int cmp_desc(const void *a, const void *b)
{
    const oc_scored *x = (const oc_scored *)a, *y = (const oc_scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}
static int cmp_asc(const void *a, const void *b)
{
    int32_t i = *(const int32_t *)a, j = *(const int32_t *)b;
    return (i > j) - (i < j);
}

int64_t oc_topk(const double *s, int64_t n, int64_t k, int32_t *idx)
{
    if (k > n) k = n;
    if (k < 0) k = 0;
    oc_scored *order = (oc_scored *)malloc(sizeof(oc_scored) * (n > 0 ? n : 1));
    for (int64_t j = 0; j < n; ++j) { order[j].s = s[j]; order[j].j = (int32_t)j; }
    qsort(order, (size_t)n, sizeof(oc_scored), cmp_desc);
    for (int64_t q = 0; q < k; ++q) idx[q] = order[q].j;
    qsort(idx, (size_t)k, sizeof(int32_t), cmp_asc);
    free(order);
    return k;
}

/* ------------------------------------------------------------------------ */
/* Gathered sparse attention for one query block.  [P2] SIP paragraph: each
 * selected block counts 1/pi times (pi = 25% counts as four blocks), the
 * Horvitz-Thompson estimator of the softmax numerator and normaliser, and it
 * is realised as a shift of the logits inside an ordinary softmax.  [P2]
 * fine-grained kernel paragraph: blocks are gathered by index, tokens keep
 * their order.  For query i:
 *   O_i = sum_{j in S} (1/pi_j) sum_{t in j} e^{a_it} v_t
 *         / sum_{j in S} (1/pi_j) sum_{t in j} e^{a_it},   a_it = scale q_i.k_t
 * evaluated as softmax over logits a_it + ln(1/pi_j).  Keys past N (ragged
 * last block) are absent.  lse_i = ln of the normaliser (natural log).  A row
 * with nothing selected returns O = 0 and lse = -inf (READING).             */
void oc_sparse_block(const double *Qb, int64_t M, const double *K, const double *V,
                     int64_t N, int64_t d, int64_t kb, const int32_t *idx,
                     const float *pi_sel, int64_t count, double scale,
                     double *O, double *lse)
{
    int64_t maxkeys = count * kb;
    double *logit = (double *)malloc(sizeof(double) * (maxkeys > 0 ? maxkeys : 1));
    int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (maxkeys > 0 ? maxkeys : 1));
    for (int64_t i = 0; i < M; ++i) {
        int64_t nk = 0;
        double m = -INFINITY;
        for (int64_t sl = 0; sl < count; ++sl) {
            double bias = log(1.0 / (double)pi_sel[sl]);
            for (int64_t t = (int64_t)idx[sl] * kb; t < ((int64_t)idx[sl] + 1) * kb && t < N; ++t) {
                double dot = 0.0;
                for (int64_t k = 0; k < d; ++k) dot += Qb[i * d + k] * K[t * d + k];
                logit[nk] = scale * dot + bias;
                key[nk] = t;
                if (logit[nk] > m) m = logit[nk];
                ++nk;
            }
        }
        for (int64_t k = 0; k < d; ++k) O[i * d + k] = 0.0;
        if (nk == 0) { lse[i] = -INFINITY; continue; }
        double den = 0.0;
        for (int64_t q = 0; q < nk; ++q) {
            double p = exp(logit[q] - m);
            den += p;
            for (int64_t k = 0; k < d; ++k) O[i * d + k] += p * V[key[q] * d + k];
        }
        for (int64_t k = 0; k < d; ++k) O[i * d + k] /= den;
        lse[i] = m + log(den);
    }
    free(logit);
    free(key);
}

/* Dense softmax attention ([P1] bottleneck section: 3D full attention).
 * Textbook softmax(scale Q K^T) V for one head; queries run in parallel.    */
void oc_dense(const double *Q, int64_t Nq, const double *K, const double *V, int64_t N,
              int64_t d, double scale, double *O, double *lse)
{
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * N);
#pragma omp for schedule(static)
        for (int64_t i = 0; i < Nq; ++i) {
            double m = -INFINITY;
            for (int64_t t = 0; t < N; ++t) {
                double dot = 0.0;
                for (int64_t k = 0; k < d; ++k) dot += Q[i * d + k] * K[t * d + k];
                logit[t] = scale * dot;
                if (logit[t] > m) m = logit[t];
            }
            double den = 0.0;
            for (int64_t k = 0; k < d; ++k) O[i * d + k] = 0.0;
            for (int64_t t = 0; t < N; ++t) {
                double p = exp(logit[t] - m);
                den += p;
                for (int64_t k = 0; k < d; ++k) O[i * d + k] += p * V[t * d + k];
            }
            for (int64_t k = 0; k < d; ++k) O[i * d + k] /= den;
            lse[i] = m + log(den);
        }
        free(logit);
    }
}

/* ------------------------------------------------------------------------ */
/* Batch drivers over rows r = (b, h, qb), b-major then h then qb.          */

/* Selector for every row: mean keys per head, k-means per q-block, scores.
 * Kbar [BH][nkvb][d], C [rows][nc][d], w [rows][nc], labels [rows][qblk],
 * S [rows][nkvb].                                                            */
void oc_selector_all(const double *Q, const double *K, int64_t BH, int64_t N, int64_t d,
                     int64_t qblk, int64_t kb, int nc, int iters, double scale,
                     double *Kbar, double *C, double *w, int32_t *labels, double *S)
{
    int64_t nqb = (N + qblk - 1) / qblk, nkvb = (N + kb - 1) / kb;
#pragma omp parallel for schedule(dynamic)
    for (int64_t bh = 0; bh < BH; ++bh)
        oc_meanpool(K + bh * N * d, N, d, kb, Kbar + bh * nkvb * d);
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < BH * nqb; ++r) {
        int64_t bh = r / nqb, qb = r % nqb;
        int64_t q0 = qb * qblk, M = (q0 + qblk < N ? q0 + qblk : N) - q0;
        oc_kmeans(Q + (bh * N + q0) * d, M, d, nc, iters, C + r * nc * d, w + r * nc,
                  labels + r * qblk);
        oc_scores(C + r * nc * d, w + r * nc, nc, Kbar + bh * nkvb * d, nkvb, d, scale,
                  S + r * nkvb);
    }
}

/* Planner for every row, mode 0 = SIP (water-fill, float32 rounding of pi,
 * Poisson sampling), mode 1 = top-k with k = floor(Bblk + 0.5).  pi_out
 * [rows][nkvb] (may be NULL), counts [rows], idx/pi_sel [rows][cap].        */
void oc_plan_all(const double *S, int64_t B, int64_t H, int64_t nqb, int64_t nkvb,
                 double Bblk, int mode, uint64_t seed, int64_t cap, float *pi_out,
                 int64_t *counts, int32_t *idx, float *pi_sel)
{
#pragma omp parallel
    {
        double *pid = (double *)malloc(sizeof(double) * nkvb);
        float *pif = (float *)malloc(sizeof(float) * nkvb);
        int32_t *tk = (int32_t *)malloc(sizeof(int32_t) * nkvb);
#pragma omp for schedule(dynamic)
        for (int64_t r = 0; r < B * H * nqb; ++r) {
            int64_t b = r / (H * nqb), h = (r / nqb) % H, qb = r % nqb;
            const double *s = S + r * nkvb;
            if (mode == 0) {
                oc_waterfill(s, nkvb, Bblk, pid, NULL);
                for (int64_t j = 0; j < nkvb; ++j) pif[j] = (float)pid[j];
                if (pi_out) memcpy(pi_out + r * nkvb, pif, sizeof(float) * nkvb);
                counts[r] = oc_sample(pif, nkvb, seed, b, h, qb, idx + r * cap, pi_sel + r * cap, cap);
            } else {
                int64_t k = (int64_t)floor(Bblk + 0.5);
                int64_t n = oc_topk(s, nkvb, k, tk);
                for (int64_t q = 0; q < n && q < cap; ++q) {
                    idx[r * cap + q] = tk[q];
                    pi_sel[r * cap + q] = 1.0f;
                }
                counts[r] = n;
            }
        }
        free(pid);
        free(pif);
        free(tk);
    }
}

/* Sparse forward for a list of rows (all rows when rows == NULL, n_rows =
 * BH * nqb).  Row r of the plan arrays belongs to flat row id rows[r].
 * O [BH][N][d] and lse [BH][N] are written only for the listed rows.        */
void oc_forward_rows(const double *Q, const double *K, const double *V, int64_t BH, int64_t N,
                     int64_t d, int64_t qblk, int64_t kb, const int64_t *rows, int64_t n_rows,
                     const int64_t *counts, const int32_t *idx, const float *pi_sel, int64_t cap,
                     double scale, double *O, double *lse)
{
    int64_t nqb = (N + qblk - 1) / qblk;
#pragma omp parallel for schedule(dynamic)
    for (int64_t q = 0; q < n_rows; ++q) {
        int64_t r = rows ? rows[q] : q;
        int64_t plan_row = rows ? q : r;
        int64_t bh = r / nqb, qb = r % nqb;
        int64_t q0 = qb * qblk, M = (q0 + qblk < N ? q0 + qblk : N) - q0;
        int64_t cnt = counts[plan_row] < cap ? counts[plan_row] : cap;
        oc_sparse_block(Q + (bh * N + q0) * d, M, K + bh * N * d, V + bh * N * d, N, d, kb,
                        idx + plan_row * cap, pi_sel + plan_row * cap, cnt, scale,
                        O + (bh * N + q0) * d, lse + bh * N + q0);
    }
}

int oc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oc_set_num_threads(int n)
{
#ifdef _OPENMP
    omp_set_num_threads(n);
#else
    (void)n;
#endif
}
