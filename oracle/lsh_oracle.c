/*
 * CPU oracle for the Reformer shared-QK LSH-attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it. It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Plain C99, fp64 throughout, no BLAS, no -ffast-math. Every loop follows the
 * definition in the order the pages state it; OpenMP only splits independent
 * (batch, head, round) units across threads and never reorders a sum.
 *
 * Sources (page title, section):
 *   [T]  "Reformer summary" (ttnews.xyz), sections 局部敏感哈希 (LSH),
 *        局部敏感哈希注意力 (LSH attention), 多輪LSH哈希 (multi-round hashing),
 *        共享QK中的自掩碼 (self-mask for shared-QK attention).
 *   [D]  "Reformer: LSH attention and reversible layers" (dtcms.com),
 *        section 二.1 (key/query normalisation; masked softmax formula).
 * Where the pages are silent (which neighbouring chunk, the round merge, tie
 * rules) the readings are stated next to the code that takes them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LSHO_SELF_LOGIT (-1.0e5)

/* ------------------------------------------------------------------------ */
/* Hash. [T] §LSH: for b buckets draw R of size [dimension, b/2] and set
 * h(x) = argmax([xR ; -xR]). The concatenation puts the b/2 projections first
 * and their negations second, so index j < b/2 is bucket j for +p_j and index
 * b/2 + j is bucket b/2 + j for -p_j. argmax returns the FIRST index that
 * attains the maximum (reading for ties).
 *
 * x: [nrows][d], R: [d][nb/2] (row-major), bucket/margin: [nrows].
 * margin = max(c) - (second largest entry of c), with ties giving 0.
 */
void lsho_hash_rows(const double *x, int64_t nrows, int d, const double *R, int nb,
                    int32_t *bucket, double *margin)
{
    const int half = nb / 2;
    double *p = (double *)malloc(sizeof(double) * (size_t)half);
    double *c = (double *)malloc(sizeof(double) * (size_t)nb);
    for (int64_t i = 0; i < nrows; ++i) {
        const double *xi = x + i * d;
        /* p_j = sum_k x_k R[k][j], summed in increasing k for every j */
        for (int j = 0; j < half; ++j) p[j] = 0.0;
        for (int k = 0; k < d; ++k) {
            const double xk = xi[k];
            const double *Rk = R + (int64_t)k * half;
            for (int j = 0; j < half; ++j) p[j] += xk * Rk[j];
        }
        for (int j = 0; j < half; ++j) {
            c[j] = p[j];
            c[half + j] = -p[j];
        }
        int best = 0;
        for (int t = 1; t < nb; ++t)
            if (c[t] > c[best]) best = t;
        double second = -INFINITY;
        for (int t = 0; t < nb; ++t)
            if (t != best && c[t] > second) second = c[t];
        bucket[i] = best;
        if (margin) margin[i] = c[best] - second;
    }
    free(p);
    free(c);
}

/* Every token of every (batch, head) against every round's R.
 * x: [BH][n][d], R: [rounds][d][nb/2] -> bucket/margin: [BH][rounds][n]. */
void lsho_hash_all(const double *x, int64_t BH, int n, int d, const double *R, int rounds, int nb,
                   int nthreads, int32_t *bucket, double *margin)
{
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t u = 0; u < BH * rounds; ++u) {
        const int64_t bh = u / rounds;
        const int r = (int)(u % rounds);
        lsho_hash_rows(x + bh * (int64_t)n * d, n, d, R + (int64_t)r * d * (nb / 2), nb,
                       bucket + u * n, margin ? margin + u * n : NULL);
    }
}

/* ------------------------------------------------------------------------ */
/* Sort. [T] §LSH attention: order the tokens by bucket, ascending, and inside
 * a bucket by position. A stable counting sort over positions 0..n-1 is
 * exactly that order. perm[s] = position held by slot s; inv[perm[s]] = s.
 * Returns 0, or -1 if a bucket id is outside [0, nb). */
int lsho_sort(const int32_t *bucket, int n, int nb, int32_t *perm, int32_t *inv)
{
    int64_t *start = (int64_t *)calloc((size_t)nb + 1, sizeof(int64_t));
    for (int i = 0; i < n; ++i) {
        if (bucket[i] < 0 || bucket[i] >= nb) {
            free(start);
            return -1;
        }
        start[bucket[i] + 1] += 1;
    }
    for (int b = 0; b < nb; ++b) start[b + 1] += start[b];
    for (int i = 0; i < n; ++i) {
        const int64_t s = start[bucket[i]]++;
        perm[s] = i;
        inv[i] = (int32_t)s;
    }
    free(start);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Chunked attention for one (batch, head, round). [T] §LSH attention: cut the
 * sorted order into groups of m and attend inside the groups; the reading
 * taken here lets a query in chunk c see the keys of chunk c and of chunk
 * c-1 (chunk 0 sees itself only; no wrap-around). A chunk size m >= n is one
 * chunk holding the whole sequence.
 *
 * Logit of query at slot s against key at slot j, positions ps = perm[s],
 * pj = perm[j]:
 *   causal and pj > ps    -> key removed (weight exactly 0)
 *   pj == ps              -> -1e5 ([T] §self-mask: a token sees itself only
 *                            when nothing else is available; the value
 *                            replaces the logit)
 *   otherwise             -> (x_ps . x_pj) / (||x_pj|| sqrt(d))
 *                            ([D] §二.1 key normalisation, scaled softmax; the
 *                            query stays un-normalised; a zero key gives 0)
 * lse = log sum_j exp(logit_j); out = sum_j softmax_j v_pj (two-pass softmax).
 *
 * x, v: [n][d] for this (batch, head). qslots: slots to evaluate (NULL = all
 * n in order). out: [nq][d], lse: [nq]. Returns 0, or -1 if n % m != 0.
 */
int lsho_attend_slots(const double *x, const double *v, const int32_t *perm, int n, int d,
                      int m, int causal, const int32_t *qslots, int64_t nq, double *out,
                      double *lse)
{
    const int mc = (m >= n) ? n : m;
    if (mc <= 0 || n % mc != 0) return -1;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    double *logit = (double *)malloc(sizeof(double) * 2 * (size_t)mc);
    int32_t *key = (int32_t *)malloc(sizeof(int32_t) * 2 * (size_t)mc);
    for (int64_t q = 0; q < nq; ++q) {
        const int s = qslots ? qslots[q] : (int)q;
        const int c = s / mc;
        const int lo = (c > 0 ? c - 1 : 0) * mc;
        const int hi = (c + 1) * mc;
        const int ps = perm[s];
        const double *xq = x + (int64_t)ps * d;
        int cnt = 0;
        for (int j = lo; j < hi; ++j) {
            const int pj = perm[j];
            if (causal && pj > ps) continue;
            double l;
            if (pj == ps) {
                l = LSHO_SELF_LOGIT;
            } else {
                const double *xk = x + (int64_t)pj * d;
                double dot = 0.0, nn = 0.0;
                for (int k = 0; k < d; ++k) {
                    dot += xq[k] * xk[k];
                    nn += xk[k] * xk[k];
                }
                const double nrm = sqrt(nn);
                l = (nrm > 0.0) ? dot / nrm * inv_sqrt_d : 0.0;
            }
            logit[cnt] = l;
            key[cnt] = pj;
            ++cnt;
        }
        /* cnt >= 1: the query's own slot is always in its window and never
         * causally removed. */
        double mx = logit[0];
        for (int t = 1; t < cnt; ++t)
            if (logit[t] > mx) mx = logit[t];
        double z = 0.0;
        for (int t = 0; t < cnt; ++t) z += exp(logit[t] - mx);
        double *o = out + q * d;
        for (int k = 0; k < d; ++k) o[k] = 0.0;
        for (int t = 0; t < cnt; ++t) {
            const double w = exp(logit[t] - mx) / z;
            const double *vk = v + (int64_t)key[t] * d;
            for (int k = 0; k < d; ++k) o[k] += w * vk[k];
        }
        lse[q] = mx + log(z);
    }
    free(logit);
    free(key);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Round merge. [T] §multi-round hashing defers the combination to the paper;
 * the reading taken: each round's normalised output is weighted by
 * exp(lse_r - logsumexp_r lse_r), which is the softmax over the union of the
 * rounds' candidate lists (duplicates counted once per round).
 * o: [rounds][npos][d], lse: [rounds][npos] -> out: [npos][d], L: [npos]. */
void lsho_merge(const double *o, const double *lse, int rounds, int64_t npos, int d, double *out,
                double *L)
{
    for (int64_t i = 0; i < npos; ++i) {
        double mx = lse[i];
        for (int r = 1; r < rounds; ++r)
            if (lse[r * npos + i] > mx) mx = lse[r * npos + i];
        double z = 0.0;
        for (int r = 0; r < rounds; ++r) z += exp(lse[r * npos + i] - mx);
        const double lsum = mx + log(z);
        double *oi = out + i * d;
        for (int k = 0; k < d; ++k) oi[k] = 0.0;
        for (int r = 0; r < rounds; ++r) {
            const double w = exp(lse[r * npos + i] - lsum);
            const double *orow = o + ((int64_t)r * npos + i) * d;
            for (int k = 0; k < d; ++k) oi[k] += w * orow[k];
        }
        if (L) L[i] = lsum;
    }
}

/* ------------------------------------------------------------------------ */
/* Whole forward pass.
 * x, v: [B][H][n][d]; R: [rounds][d][nb/2]; buckets_in: [B][H][rounds][n] or
 * NULL (hash here). Outputs in position order: out [B][H][n][d], lse
 * [B][H][rounds][n], buckets_out [B][H][rounds][n] (may be NULL).
 * nthreads <= 0 uses the OpenMP default. Returns 0 or a negative error. */
int lsho_forward(const double *x, const double *v, const double *R, const int32_t *buckets_in,
                 int B, int H, int n, int d, int nb, int m, int rounds, int causal, int nthreads,
                 double *out, double *lse, int32_t *buckets_out)
{
    const int mc = (m >= n) ? n : m;
    if (mc <= 0 || n % mc != 0 || nb < 2 || nb % 2 != 0) return -1;
    const int64_t units = (int64_t)B * H * rounds;
    const int64_t nd = (int64_t)n * d;
    double *o_all = (double *)malloc(sizeof(double) * (size_t)(units * nd));
    int32_t *bk_all = (int32_t *)malloc(sizeof(int32_t) * (size_t)(units * n));
    if (!o_all || !bk_all) {
        free(o_all);
        free(bk_all);
        return -2;
    }
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : err)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t bh = u / rounds;
        const int r = (int)(u % rounds);
        const double *xs = x + bh * nd;
        const double *vs = v + bh * nd;
        int32_t *bk = bk_all + u * n;
        if (buckets_in) {
            memcpy(bk, buckets_in + u * n, sizeof(int32_t) * (size_t)n);
        } else {
            lsho_hash_rows(xs, n, d, R + (int64_t)r * d * (nb / 2), nb, bk, NULL);
        }
        int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        double *os = (double *)malloc(sizeof(double) * (size_t)nd);
        double *ls = (double *)malloc(sizeof(double) * (size_t)n);
        if (lsho_sort(bk, n, nb, perm, inv) != 0) {
            err |= 1;
        } else {
            lsho_attend_slots(xs, vs, perm, n, d, m, causal, NULL, n, os, ls);
            /* undo the sort: position i takes slot inv[i] */
            double *od = o_all + u * nd;
            for (int i = 0; i < n; ++i) {
                memcpy(od + (int64_t)i * d, os + (int64_t)inv[i] * d, sizeof(double) * (size_t)d);
                lse[u * n + i] = ls[inv[i]];
            }
        }
        free(perm);
        free(inv);
        free(os);
        free(ls);
    }
    if (err) {
        free(o_all);
        free(bk_all);
        return -3;
    }
    /* merge rounds for every (b, h) */
    const int64_t BH = (int64_t)B * H;
#ifdef _OPENMP
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t bh = 0; bh < BH; ++bh)
        lsho_merge(o_all + bh * rounds * nd, lse + bh * rounds * n, rounds, n, d, out + bh * nd,
                   NULL);
    if (buckets_out) memcpy(buckets_out, bk_all, sizeof(int32_t) * (size_t)(units * n));
    free(o_all);
    free(bk_all);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The forward pass evaluated at a sample of positions only, with given
 * buckets (the sort still runs over the whole sequence, since a position's
 * chunk depends on every bucket id). pos: [npos] positions, the same for
 * every (b, h). out: [B][H][npos][d], lse: [B][H][rounds][npos]. */
int lsho_forward_sampled(const double *x, const double *v, const int32_t *buckets, int B, int H,
                         int n, int d, int nb, int m, int rounds, int causal, const int32_t *pos,
                         int npos, int nthreads, double *out, double *lse)
{
    const int mc = (m >= n) ? n : m;
    if (mc <= 0 || n % mc != 0) return -1;
    const int64_t BH = (int64_t)B * H;
    const int64_t nd = (int64_t)n * d;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : err)
#endif
    for (int64_t bh = 0; bh < BH; ++bh) {
        int32_t *perm = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        int32_t *inv = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        int32_t *qs = (int32_t *)malloc(sizeof(int32_t) * (size_t)npos);
        double *o = (double *)malloc(sizeof(double) * (size_t)rounds * npos * d);
        double *l = lse + bh * rounds * npos;
        for (int r = 0; r < rounds && !err; ++r) {
            if (lsho_sort(buckets + (bh * rounds + r) * n, n, nb, perm, inv) != 0) {
                err |= 1;
                break;
            }
            for (int t = 0; t < npos; ++t) qs[t] = inv[pos[t]];
            lsho_attend_slots(x + bh * nd, v + bh * nd, perm, n, d, m, causal, qs, npos,
                              o + (int64_t)r * npos * d, l + (int64_t)r * npos);
        }
        if (!err) lsho_merge(o, l, rounds, npos, d, out + bh * npos * d, NULL);
        free(perm);
        free(inv);
        free(qs);
        free(o);
    }
    return err ? -3 : 0;
}
