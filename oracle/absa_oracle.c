/*
 * absa_oracle.c -- plain, slow CPU reference of the AB-Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, by the package smoke check
 * and by the benchmark's CPU-baseline leg, never by the product path.
 * Every function follows one step of the method as the AB-Attention summary
 * page states it (section "AB-Attention's three techniques": the IBCS, SIP and
 * 4-token-block paragraphs); the readings of what the page leaves open are
 * written in absa_oracle.h beside each declaration.
 *
 * Parity status: every function here is pinned by the oracle self-tests
 * (closed forms, invariants, library routines, brute force, the page's
 * 25%-counts-as-four example); the whole-op composition has no printed
 * example values to pin against.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 * -ffp-contract=off keeps every fp32 operation of the k-means exactly as
 * written (the only fused multiply-adds are the explicit fmaf calls).
 */
#include "absa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

float oracle_bf16_to_float(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* ---------------------------------------------------------------- pooling */

void oracle_pool_keys(const uint16_t *k, int64_t N, int d, double *kbar)
{
    int64_t nkb = (N + 3) / 4;
    for (int64_t j = 0; j < nkb; ++j) {
        int64_t t0 = 4 * j;
        int64_t t1 = t0 + 4 < N ? t0 + 4 : N;
        for (int e = 0; e < d; ++e) {
            double sum = 0.0;
            for (int64_t t = t0; t < t1; ++t)
                sum += (double)oracle_bf16_to_float(k[t * d + e]);
            kbar[j * d + e] = sum / (double)(t1 - t0);
        }
    }
}

/* ---------------------------------------------------------------- k-means */

void oracle_kmeans_block(const uint16_t *q, int m, int d, int nc, int iters,
                         float *mu, float *w, int32_t *assign, int32_t *count)
{
    float *x = (float *)malloc(sizeof(float) * (size_t)m * d);
    float *sum = (float *)malloc(sizeof(float) * (size_t)nc * d);
    for (int i = 0; i < m; ++i)
        for (int e = 0; e < d; ++e)
            x[i * d + e] = oracle_bf16_to_float(q[(size_t)i * d + e]);

    /* initial centroids: the queries at offsets floor(c*m/nc) */
    for (int c = 0; c < nc; ++c) {
        int i0 = (int)(((int64_t)c * m) / nc);
        for (int e = 0; e < d; ++e)
            mu[c * d + e] = x[i0 * d + e];
    }

    for (int it = 0; it < iters; ++it) {
        /* assignment: nearest centroid, ties to the lowest index */
        for (int i = 0; i < m; ++i) {
            int best = 0;
            float best_dist = 0.0f;
            for (int c = 0; c < nc; ++c) {
                float dist = 0.0f;
                for (int e = 0; e < d; ++e) {
                    float diff = x[i * d + e] - mu[c * d + e];
                    dist = fmaf(diff, diff, dist);
                }
                if (c == 0 || dist < best_dist) {
                    best = c;
                    best_dist = dist;
                }
            }
            assign[i] = best;
        }
        /* update: mean of the members; an empty cluster keeps its centroid */
        for (int c = 0; c < nc; ++c) {
            count[c] = 0;
            for (int e = 0; e < d; ++e)
                sum[c * d + e] = 0.0f;
        }
        for (int i = 0; i < m; ++i) {
            int c = assign[i];
            count[c] += 1;
            for (int e = 0; e < d; ++e)
                sum[c * d + e] = sum[c * d + e] + x[i * d + e];
        }
        for (int c = 0; c < nc; ++c) {
            if (count[c] == 0)
                continue;
            for (int e = 0; e < d; ++e)
                mu[c * d + e] = sum[c * d + e] / (float)count[c];
        }
    }
    /* weight = share of the block's queries in the cluster (last assignment) */
    for (int c = 0; c < nc; ++c)
        w[c] = (float)count[c] / (float)m;
    free(x);
    free(sum);
}

/* ----------------------------------------------------------------- scores */

void oracle_block_scores(const float *mu, const float *w, int nc, int d,
                         const double *kbar, int nkb, double scale, double *s)
{
    double *logit = (double *)malloc(sizeof(double) * (size_t)nkb);
    for (int j = 0; j < nkb; ++j)
        s[j] = 0.0;
    for (int c = 0; c < nc; ++c) {
        if (!(w[c] > 0.0f))
            continue;
        double mx = -INFINITY;
        for (int j = 0; j < nkb; ++j) {
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)mu[c * d + e] * kbar[(size_t)j * d + e];
            logit[j] = scale * dot;
            if (logit[j] > mx)
                mx = logit[j];
        }
        double z = 0.0;
        for (int j = 0; j < nkb; ++j)
            z += exp(logit[j] - mx);
        for (int j = 0; j < nkb; ++j)
            s[j] += (double)w[c] * exp(logit[j] - mx) / z;
    }
    free(logit);
}

/* --------------------------------------------------------------- SIP: pi */

#define TWO32 4294967296.0

static uint64_t quantised_score(float s)
{
    /* q = max(1, floor(s * 2^32)), NaN/negative -> 1, at most 2^32 */
    double x = (double)s * TWO32;
    if (!(x >= 1.0))
        return 1u;
    if (x >= TWO32)
        return (uint64_t)1 << 32;
    return (uint64_t)x; /* truncation == floor for x >= 1 */
}

int oracle_pi_solve(const float *s, int nkb, int64_t n, uint8_t *capped,
                    uint64_t *r_out, uint64_t *R_out)
{
    memset(capped, 0, (size_t)nkb);
    int rounds = 0;
    for (;;) {
        int64_t n_capped = 0;
        uint64_t R = 0;
        for (int j = 0; j < nkb; ++j) {
            if (capped[j])
                n_capped += 1;
            else
                R += quantised_score(s[j]);
        }
        uint64_t r = (uint64_t)(n - n_capped);
        int grew = 0;
        for (int j = 0; j < nkb; ++j) {
            if (!capped[j] && r * quantised_score(s[j]) >= R) {
                capped[j] = 1;
                grew = 1;
            }
        }
        rounds += 1;
        if (!grew) {
            *r_out = r;
            *R_out = R;
            return rounds;
        }
    }
}

/* ------------------------------------------------------------- SIP: draws */

uint64_t oracle_splitmix64_mix(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint32_t oracle_draw_u32(uint64_t seed, uint64_t ctr)
{
    /* output number ctr+1 of SplitMix64 started from state key = mix(seed) */
    uint64_t key = oracle_splitmix64_mix(seed);
    uint64_t z = oracle_splitmix64_mix(key + (ctr + 1) * 0x9E3779B97F4A7C15ull);
    return (uint32_t)(z >> 32);
}

int oracle_sample_row(const float *s, int nkb, int64_t n, uint64_t seed,
                      uint64_t row, int cap, int32_t *kv_index, float *log_pi,
                      uint64_t *r_out, uint64_t *R_out)
{
    if (n >= nkb) {
        for (int j = 0; j < nkb && j < cap; ++j) {
            kv_index[j] = j;
            log_pi[j] = 0.0f;
        }
        *r_out = 0;
        *R_out = 0;
        return nkb;
    }
    uint8_t *capped = (uint8_t *)malloc((size_t)nkb);
    uint64_t r, R;
    oracle_pi_solve(s, nkb, n, capped, &r, &R);
    int taken = 0;
    for (int j = 0; j < nkb; ++j) {
        int take;
        uint64_t rq = 0;
        if (capped[j]) {
            take = 1;
        } else {
            rq = r * quantised_score(s[j]);
            unsigned __int128 lhs =
                (unsigned __int128)oracle_draw_u32(seed, row * (uint64_t)nkb + (uint64_t)j) * R;
            unsigned __int128 rhs = (unsigned __int128)rq << 32;
            take = lhs < rhs;
        }
        if (take) {
            if (taken < cap) {
                kv_index[taken] = j;
                log_pi[taken] = capped[j] ? 0.0f : (float)log((double)rq / (double)R);
            }
            taken += 1;
        }
    }
    free(capped);
    *r_out = r;
    *R_out = R;
    return taken;
}

/* Systematic (fixed-size) design, written from its definition: with the
 * integer pi of oracle_pi_solve scaled by R (a_j = R if capped, r*q_j
 * otherwise; sum a_j = n*R), lay the blocks end to end on [0, n*R) in
 * ascending j and put n points at (k + U/2^32)*R, k = 0..n-1.  Block j is
 * taken iff a point falls in its interval [A_j, A_j + a_j), A_j = sum_{i<j} a_i.
 * Each interval is at most R long, so it holds at most one point, block j is
 * taken with probability a_j/R = pi_j over U, and exactly n blocks are taken.
 * Arithmetic in units of R/2^32: point k sits at k*R*2^32 + U*R. */
int oracle_systematic_take(const float *s, int nkb, int64_t n, uint32_t U,
                           uint8_t *take, uint64_t *r_out, uint64_t *R_out)
{
    uint8_t *capped = (uint8_t *)malloc((size_t)nkb);
    uint64_t r, R;
    oracle_pi_solve(s, nkb, n, capped, &r, &R);
    const unsigned __int128 period = (unsigned __int128)R << 32;
    const unsigned __int128 phase = (unsigned __int128)U * R;
    unsigned __int128 A = 0;  /* A_j * 2^32 */
    int taken = 0;
    for (int j = 0; j < nkb; ++j) {
        const uint64_t a = capped[j] ? R : r * quantised_score(s[j]);
        const unsigned __int128 lo = A, hi = A + ((unsigned __int128)a << 32);
        /* first point at or after lo: k0 = ceil((lo - phase) / period) */
        unsigned __int128 k0 = 0;
        if (lo > phase)
            k0 = (lo - phase + period - 1) / period;
        take[j] = (k0 < (unsigned __int128)n) && (k0 * period + phase < hi);
        taken += take[j];
        A = hi;
    }
    free(capped);
    *r_out = r;
    *R_out = R;
    return taken;
}

int oracle_sample_row_systematic(const float *s, int nkb, int64_t n, uint64_t seed,
                                 uint64_t row, int cap, int32_t *kv_index, float *log_pi,
                                 uint64_t *r_out, uint64_t *R_out)
{
    if (n >= nkb)
        return oracle_sample_row(s, nkb, n, seed, row, cap, kv_index, log_pi, r_out, R_out);
    uint8_t *take = (uint8_t *)malloc((size_t)nkb);
    uint64_t r, R;
    const uint32_t U = oracle_draw_u32(seed, row * (uint64_t)nkb);
    oracle_systematic_take(s, nkb, n, U, take, &r, &R);
    int taken = 0;
    for (int j = 0; j < nkb; ++j) {
        if (!take[j])
            continue;
        if (taken < cap) {
            const uint64_t rq = r * quantised_score(s[j]);
            kv_index[taken] = j;
            log_pi[taken] = rq >= R ? 0.0f : (float)log((double)rq / (double)R);
        }
        taken += 1;
    }
    free(take);
    *r_out = r;
    *R_out = R;
    return taken;
}

/* -------------------------------------------------------------- attention */

static void attention_row(const float *qf, int d, const uint16_t *k,
                          const uint16_t *v, int64_t N, const int32_t *blocks,
                          const float *log_pi, int count, double scale,
                          int have_mref, double m_ref, double *num, double *den)
{
    /* pass 1: logits and their max */
    int64_t ntok = 0;
    for (int b = 0; b < count; ++b)
        for (int t = 0; t < 4; ++t)
            if (4 * (int64_t)blocks[b] + t < N)
                ntok += 1;
    double *l = (double *)malloc(sizeof(double) * (size_t)(ntok > 0 ? ntok : 1));
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(ntok > 0 ? ntok : 1));
    int64_t p = 0;
    double mx = -INFINITY;
    for (int b = 0; b < count; ++b) {
        for (int t = 0; t < 4; ++t) {
            int64_t n = 4 * (int64_t)blocks[b] + t;
            if (n >= N)
                continue;
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)qf[e] * (double)oracle_bf16_to_float(k[n * d + e]);
            l[p] = scale * dot - (double)log_pi[b];
            tok[p] = n;
            if (l[p] > mx)
                mx = l[p];
            p += 1;
        }
    }
    if (have_mref)
        mx = m_ref;
    for (int e = 0; e < d; ++e)
        num[e] = 0.0;
    *den = 0.0;
    for (int64_t i = 0; i < ntok; ++i) {
        double pw = exp(l[i] - mx);
        *den += pw;
        for (int e = 0; e < d; ++e)
            num[e] += pw * (double)oracle_bf16_to_float(v[tok[i] * d + e]);
    }
    free(l);
    free(tok);
}

void oracle_sparse_attention_rows(const uint16_t *q, int nrows, int d,
                                  const uint16_t *k, const uint16_t *v,
                                  int64_t N, const int32_t *blocks,
                                  const float *log_pi, int count, double scale,
                                  double *o)
{
    float *qf = (float *)malloc(sizeof(float) * (size_t)d);
    double *num = (double *)malloc(sizeof(double) * (size_t)d);
    for (int r = 0; r < nrows; ++r) {
        for (int e = 0; e < d; ++e)
            qf[e] = oracle_bf16_to_float(q[(size_t)r * d + e]);
        double den;
        attention_row(qf, d, k, v, N, blocks, log_pi, count, scale, 0, 0.0, num, &den);
        for (int e = 0; e < d; ++e)
            o[(size_t)r * d + e] = den > 0.0 ? num[e] / den : 0.0;
    }
    free(qf);
    free(num);
}

/* ESTRA-style remainder (ESTRA page, summary and figure: cluster, compute the
 * selected pairs exactly, approximate the rest from group averages with a
 * variance-calibrated mean correction).  Reading: the listed blocks are the
 * exact part (no ln pi shift); the keys are grouped into runs of
 * `group_blocks` consecutive 4-token blocks; every group g contributes one
 * representative with the mean key mu_g and mean value nu_g of its tokens,
 * weight m_g = tokens of g not in the listed blocks, and the correction of
 * the mean for the spread of the keys taken as isotropic:
 *   sum_{t in rest of g} exp(s q.k_t) ~ m_g exp(s q.mu_g + s^2 |q|^2 var_g / 2),
 * var_g = (1/d) sum_e (mean_t k_te^2 - mu_ge^2)  (the identity
 * E exp(X) = exp(E X + Var X / 2) of a Gaussian X = s q.k).  One softmax
 * runs over the exact tokens and the representatives together. */
void oracle_remainder_attention_rows(const uint16_t *q, int nrows, int d,
                                     const uint16_t *k, const uint16_t *v,
                                     int64_t N, const int32_t *blocks, int count,
                                     int group_blocks, double scale, double *o)
{
    const int64_t nkb = (N + 3) / 4;
    const int64_t ng = (nkb + group_blocks - 1) / group_blocks;
    double *mu = (double *)calloc((size_t)(ng * d), sizeof(double));
    double *nu = (double *)calloc((size_t)(ng * d), sizeof(double));
    double *var = (double *)calloc((size_t)ng, sizeof(double));
    double *rest = (double *)calloc((size_t)ng, sizeof(double));
    double *sq = (double *)malloc(sizeof(double) * (size_t)d);
    /* group statistics over all tokens of each group */
    for (int64_t g = 0; g < ng; ++g) {
        const int64_t t0 = 4 * g * group_blocks;
        int64_t t1 = t0 + 4 * (int64_t)group_blocks;
        if (t1 > N)
            t1 = N;
        const double n = (double)(t1 - t0);
        for (int e = 0; e < d; ++e)
            sq[e] = 0.0;
        for (int64_t t = t0; t < t1; ++t)
            for (int e = 0; e < d; ++e) {
                const double kv = (double)oracle_bf16_to_float(k[t * d + e]);
                mu[g * d + e] += kv;
                sq[e] += kv * kv;
                nu[g * d + e] += (double)oracle_bf16_to_float(v[t * d + e]);
            }
        double vs = 0.0;
        for (int e = 0; e < d; ++e) {
            mu[g * d + e] /= n;
            nu[g * d + e] /= n;
            double ve = sq[e] / n - mu[g * d + e] * mu[g * d + e];
            vs += ve > 0.0 ? ve : 0.0;
        }
        var[g] = vs / (double)d;
        rest[g] = n;
    }
    /* tokens of the listed blocks leave their group's rest */
    for (int b = 0; b < count; ++b) {
        const int64_t j = blocks[b];
        if (j < 0 || j >= nkb)
            continue;
        int64_t ntok = N - 4 * j;
        if (ntok > 4)
            ntok = 4;
        rest[j / group_blocks] -= (double)ntok;
    }
    const int64_t ntok_exact = 4 * (int64_t)(count > 0 ? count : 1);
    double *l = (double *)malloc(sizeof(double) * (size_t)(ntok_exact + ng));
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)ntok_exact);
    float *qf = (float *)malloc(sizeof(float) * (size_t)d);
    for (int r = 0; r < nrows; ++r) {
        double qq = 0.0;
        for (int e = 0; e < d; ++e) {
            qf[e] = oracle_bf16_to_float(q[(size_t)r * d + e]);
            qq += (double)qf[e] * (double)qf[e];
        }
        double mx = -INFINITY;
        int64_t p = 0;
        for (int b = 0; b < count; ++b)
            for (int t = 0; t < 4; ++t) {
                const int64_t n = 4 * (int64_t)blocks[b] + t;
                if (blocks[b] < 0 || n >= N)
                    continue;
                double dot = 0.0;
                for (int e = 0; e < d; ++e)
                    dot += (double)qf[e] * (double)oracle_bf16_to_float(k[n * d + e]);
                l[p] = scale * dot;
                tok[p] = n;
                if (l[p] > mx)
                    mx = l[p];
                p += 1;
            }
        for (int64_t g = 0; g < ng; ++g) {
            double *lg = &l[p + g];
            if (rest[g] <= 0.0) {
                *lg = -INFINITY;
                continue;
            }
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)qf[e] * mu[g * d + e];
            *lg = scale * dot + 0.5 * scale * scale * qq * var[g] + log(rest[g]);
            if (*lg > mx)
                mx = *lg;
        }
        double den = 0.0;
        for (int e = 0; e < d; ++e)
            o[(size_t)r * d + e] = 0.0;
        for (int64_t i = 0; i < p; ++i) {
            const double w = exp(l[i] - mx);
            den += w;
            for (int e = 0; e < d; ++e)
                o[(size_t)r * d + e] += w * (double)oracle_bf16_to_float(v[tok[i] * d + e]);
        }
        for (int64_t g = 0; g < ng; ++g) {
            if (l[p + g] == -INFINITY)
                continue;
            const double w = exp(l[p + g] - mx);
            den += w;
            for (int e = 0; e < d; ++e)
                o[(size_t)r * d + e] += w * nu[g * d + e];
        }
        for (int e = 0; e < d; ++e)
            o[(size_t)r * d + e] = den > 0.0 ? o[(size_t)r * d + e] / den : 0.0;
    }
    free(mu);
    free(nu);
    free(var);
    free(rest);
    free(sq);
    free(l);
    free(tok);
    free(qf);
}

void oracle_dense_attention_rows(const uint16_t *q, int nrows, int d,
                                 const uint16_t *k, const uint16_t *v,
                                 int64_t N, double scale, double *o)
{
    /* a plain loop over every token, written apart from the sparse path */
    double *l = (double *)malloc(sizeof(double) * (size_t)N);
    for (int r = 0; r < nrows; ++r) {
        double mx = -INFINITY;
        for (int64_t n = 0; n < N; ++n) {
            double dot = 0.0;
            for (int e = 0; e < d; ++e)
                dot += (double)oracle_bf16_to_float(q[(size_t)r * d + e]) *
                       (double)oracle_bf16_to_float(k[n * d + e]);
            l[n] = scale * dot;
            if (l[n] > mx)
                mx = l[n];
        }
        double den = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            l[n] = exp(l[n] - mx);
            den += l[n];
        }
        for (int e = 0; e < d; ++e) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                acc += l[n] * (double)oracle_bf16_to_float(v[n * d + e]);
            o[(size_t)r * d + e] = acc / den;
        }
    }
    free(l);
}

void oracle_ht_parts(const uint16_t *q, int d, const uint16_t *k,
                     const uint16_t *v, int64_t N, const int32_t *blocks,
                     const float *log_pi, int count, double scale,
                     double m_ref, double *nhat, double *dhat)
{
    float *qf = (float *)malloc(sizeof(float) * (size_t)d);
    for (int e = 0; e < d; ++e)
        qf[e] = oracle_bf16_to_float(q[e]);
    attention_row(qf, d, k, v, N, blocks, log_pi, count, scale, 1, m_ref, nhat, dhat);
    free(qf);
}

/* ------------------------------------------------------ whole-layer drivers */

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_select_scores(int B, int H, int64_t N, int d, int nc, int iters,
                          double scale, const uint16_t *q, const uint16_t *k,
                          int qb_lo, int qb_hi, float *scores, float *mu,
                          float *w, int32_t *assign)
{
    int nqb = (int)((N + 127) / 128);
    int nkb = (int)((N + 3) / 4);
    if (qb_hi <= 0 || qb_hi > nqb)
        qb_hi = nqb;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        const uint16_t *qh = q + (size_t)bh * N * d;
        const uint16_t *kh = k + (size_t)bh * N * d;
        double *kbar = (double *)malloc(sizeof(double) * (size_t)nkb * d);
        double *s = (double *)malloc(sizeof(double) * (size_t)nkb);
        int32_t count[64];
        oracle_pool_keys(kh, N, d, kbar);
        for (int qb = qb_lo; qb < qb_hi; ++qb) {
            size_t row = (size_t)bh * nqb + qb;
            int64_t n0 = (int64_t)qb * 128;
            int m = (int)(N - n0 < 128 ? N - n0 : 128);
            float *mu_r = mu + row * nc * d;
            float *w_r = w + row * nc;
            int32_t *as = assign + row * 128;
            for (int i = m; i < 128; ++i)
                as[i] = -1;
            oracle_kmeans_block(qh + n0 * d, m, d, nc, iters, mu_r, w_r, as, count);
            oracle_block_scores(mu_r, w_r, nc, d, kbar, nkb, scale, s);
            for (int j = 0; j < nkb; ++j)
                scores[row * nkb + j] = (float)s[j];
        }
        free(kbar);
        free(s);
    }
}

int oracle_sample_plan_design(int B, int H, int nqb, int nkb, int64_t n,
                              uint64_t seed, const float *scores, int cap,
                              int32_t *counts, int32_t *kv_index, float *log_pi,
                              uint64_t *r_R, int design)
{
    int overflow = 0;
    int64_t rows = (int64_t)B * H * nqb;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : overflow)
    for (int64_t row = 0; row < rows; ++row) {
        uint64_t r, R;
        /* paired design: the draws of row (b,h,qb) are those of (b,h,qb with
         * its low bit cleared) */
        const int64_t draw_row = design == 2 ? row - ((row % nqb) & 1) : row;
        int taken = (design == 1 ? oracle_sample_row_systematic : oracle_sample_row)(
            scores + row * nkb, nkb, n, seed, (uint64_t)draw_row, cap, kv_index + row * cap,
            log_pi + row * cap, &r, &R);
        counts[row] = taken < cap ? taken : cap;
        r_R[2 * row] = r;
        r_R[2 * row + 1] = R;
        if (taken > cap)
            overflow += 1;
    }
    return overflow;
}

int oracle_sample_plan(int B, int H, int nqb, int nkb, int64_t n, uint64_t seed,
                       const float *scores, int cap, int32_t *counts, int32_t *kv_index,
                       float *log_pi, uint64_t *r_R)
{
    return oracle_sample_plan_design(B, H, nqb, nkb, n, seed, scores, cap, counts, kv_index,
                                     log_pi, r_R, 0);
}

void oracle_sparse_attention(int B, int H, int64_t N, int d, double scale,
                             const uint16_t *q, const uint16_t *k,
                             const uint16_t *v, int nqb, int cap,
                             const int32_t *counts, const int32_t *kv_index,
                             const float *log_pi, int qb_lo, int qb_hi,
                             double *o)
{
    if (qb_hi <= 0 || qb_hi > nqb)
        qb_hi = nqb;
    int nsel = qb_hi - qb_lo;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t item = 0; item < (int64_t)B * H * nsel; ++item) {
        int64_t bh = item / nsel;
        int qb = qb_lo + (int)(item % nsel);
        size_t row = (size_t)bh * nqb + qb;
        int64_t n0 = (int64_t)qb * 128;
        int m = (int)(N - n0 < 128 ? N - n0 : 128);
        oracle_sparse_attention_rows(q + ((size_t)bh * N + n0) * d, m, d,
                                     k + (size_t)bh * N * d, v + (size_t)bh * N * d, N,
                                     kv_index + row * cap, log_pi + row * cap,
                                     counts[row], scale, o + ((size_t)bh * N + n0) * d);
    }
}
