/*
 * absa_oracle.h -- plain CPU reference of the AB-Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  The CUDA library
 * shares no code, header, table or constant with it.
 *
 * Source of every step: the AB-Attention summary page (news.hamidun.com,
 * "AB-Attention speeds up video generation by up to 2.23x and skips 92% of
 * attention"), section "AB-Attention's three techniques":
 *   - IBCS paragraph: 128-query blocks, 8 clusters per block, centroid weight
 *     = share of the block's queries, block score = weighted attention of the
 *     centroids to the block's averaged keys, original token order kept.
 *   - SIP paragraph: inclusion probability proportional to score, top blocks
 *     always taken, every block a nonzero chance, selected block weighted by
 *     1/pi (a 25% block counts as four), ordinary softmax with a logit shift.
 *   - third paragraph: 4-token key/value blocks; plan recomputed every four
 *     denoising steps while attention runs every step.
 * Readings of the points those paragraphs leave open (distance, empty
 * clusters, integer pi solve, hash, Poisson design) are stated beside each
 * function below.
 *
 * Precision: fp64 everywhere except the k-means, whose argmin decisions are
 * taken in fp32 (the precision of the GPU selector), with the arithmetic
 * order spelled out so that both sides reach the same decisions.
 * Inputs q, k, v are bf16 bit patterns (uint16), widened exactly.
 */
#ifndef ABSA_ORACLE_H
#define ABSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Widen one bf16 bit pattern to float (exact). */
float oracle_bf16_to_float(uint16_t h);

/* IBCS "averaged keys": kbar[j][e] = mean of k[t][e] over the tokens t of
 * 4-token block j (t = 4j..4j+3, clipped at N).  k is [N][d] for one (b,h);
 * kbar is [ceil(N/4)][d], fp64. */
void oracle_pool_keys(const uint16_t *k, int64_t N, int d, double *kbar);

/* IBCS intra-block k-means for one query block of m valid queries (rows of
 * q, [m][d]).  Reading: squared Euclidean distance on the raw queries;
 * initial centroids mu_c = x[floor(c*m/nc)]; `iters` Lloyd rounds, each an
 * assignment (argmin, ties to the lowest c) followed by an update (mean of the
 * members; an empty cluster keeps its centroid); weights from the last
 * assignment, w_c = |c| / m.
 * fp32 arithmetic, in this order: distance accumulated over ascending e with
 * fused multiply-add of (x - mu); member sums accumulated over ascending i
 * with round-to-nearest adds; mu = sum / count, correctly rounded.
 * Outputs: mu [nc][d], w [nc], assign [m], count [nc]. */
void oracle_kmeans_block(const uint16_t *q, int m, int d, int nc, int iters,
                         float *mu, float *w, int32_t *assign, int32_t *count);

/* IBCS block score for one query block: for each centroid c with w_c > 0,
 * l_cj = scale * (mu_c . kbar_j); a_c = softmax over all nkb blocks;
 * s_j = sum_c w_c a_cj.  fp64; s is [nkb]. */
void oracle_block_scores(const float *mu, const float *w, int nc, int d,
                         const double *kbar, int nkb, double scale, double *s);

/* SIP inclusion probabilities for one row of scores (fp32, as the score
 * array is stored).  Reading: q_j = max(1, floor(s_j * 2^32)) (NaN or
 * negative -> 1, capped at 2^32); starting from C = {} repeat
 * r = n - |C|, R = sum_{j not in C} q_j, C += {j not in C : r*q_j >= R}
 * until C stops growing.  Then pi_j = 1 on C, r*q_j/R elsewhere, and
 * sum pi = n exactly.  Requires 1 <= n < nkb.  Outputs capped[nkb] (0/1),
 * *r_out, *R_out; returns the number of capping rounds. */
int oracle_pi_solve(const float *s, int nkb, int64_t n, uint8_t *capped,
                    uint64_t *r_out, uint64_t *R_out);

/* SplitMix64 output function (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014). */
uint64_t oracle_splitmix64_mix(uint64_t z);

/* Counter-based uniform for the SIP draw of block j of row `row`:
 * ctr = row*nkb + j; u = high 32 bits of output number ctr+1 of the
 * SplitMix64 generator started from state key = mix(seed), i.e.
 * u = mix(key + (ctr+1) * 0x9E3779B97F4A7C15) >> 32 (mod 2^64 arithmetic).
 * mix(0) = 0, so seed 0 gives the published SplitMix64 stream from state 0. */
uint32_t oracle_draw_u32(uint64_t seed, uint64_t ctr);

/* SIP plan for one row (b,h,qb) whose flat index is `row`
 * (((b*H + h)*NQB + qb)).  n >= nkb: every block, log_pi = 0, r = R = 0.
 * Else Poisson sampling: block j is taken iff capped, or
 * u_j * R < (r*q_j) * 2^32 (128-bit compare).  Taken blocks are written in
 * ascending j with log_pi = 0 (capped) or (float)log((double)(r*q_j)/R).
 * At most `cap` entries are written; returns the number of taken blocks
 * (which may exceed cap: the caller treats that as overflow). */
int oracle_sample_row(const float *s, int nkb, int64_t n, uint64_t seed,
                      uint64_t row, int cap, int32_t *kv_index, float *log_pi,
                      uint64_t *r_out, uint64_t *R_out);

/* Fixed-size alternative to the Poisson design (the SIP paragraph names no
 * design): systematic sampling with probabilities pi.  Reading: the blocks
 * are laid end to end in ascending j with lengths a_j = pi_j * R (a_j = R
 * if capped, r*q_j otherwise), n points are placed at (k + U/2^32) * R for
 * k = 0..n-1, and block j is taken iff a point falls in its interval.  Each
 * block is taken with probability pi_j over U and exactly n blocks are
 * taken.  take[nkb] (0/1); returns the number taken.  Requires
 * 1 <= n < nkb. */
int oracle_systematic_take(const float *s, int nkb, int64_t n, uint32_t U,
                           uint8_t *take, uint64_t *r_out, uint64_t *R_out);

/* Plan row of the systematic design: U = oracle_draw_u32(seed, row*nkb)
 * (the counter of block 0 of the row), entries and log_pi as in
 * oracle_sample_row; n >= nkb takes every block. */
int oracle_sample_row_systematic(const float *s, int nkb, int64_t n, uint64_t seed,
                                 uint64_t row, int cap, int32_t *kv_index, float *log_pi,
                                 uint64_t *r_out, uint64_t *R_out);

/* Horvitz-Thompson sparse attention for `nrows` query rows (bf16, [nrows][d])
 * of one (b,h) over the tokens of the listed 4-token blocks (ascending), with
 * logit l_t = scale*(q.k_t) - log_pi[block of t]:
 * o = sum softmax(l)_t v_t; an empty block list gives o = 0.  k, v are [N][d]
 * for the head.  fp64 output o [nrows][d]. */
void oracle_sparse_attention_rows(const uint16_t *q, int nrows, int d,
                                  const uint16_t *k, const uint16_t *v,
                                  int64_t N, const int32_t *blocks,
                                  const float *log_pi, int count, double scale,
                                  double *o);

/* Dense softmax attention for `nrows` query rows over all N tokens of the
 * head: the full-attention reference of the evaluation section.  fp64. */
/* ESTRA-style remainder attention of query rows q [nrows,d] of one head:
 * the listed blocks exactly (no ln pi shift), every group of group_blocks
 * consecutive 4-token blocks as one representative (mean key, mean value,
 * weight = its tokens outside the listed blocks, log-weight corrected by
 * s^2 |q|^2 var_g / 2 with var_g the per-dimension key variance averaged
 * over dimensions); one softmax over both.  o is fp64 [nrows,d]. */
void oracle_remainder_attention_rows(const uint16_t *q, int nrows, int d,
                                     const uint16_t *k, const uint16_t *v,
                                     int64_t N, const int32_t *blocks, int count,
                                     int group_blocks, double scale, double *o);

void oracle_dense_attention_rows(const uint16_t *q, int nrows, int d,
                                 const uint16_t *k, const uint16_t *v,
                                 int64_t N, double scale, double *o);

/* Unnormalised HT parts for one query row: with a caller-given reference
 * max m_ref, Nhat = sum_t exp(l_t - m_ref) v_t and Dhat = sum_t
 * exp(l_t - m_ref), l_t as in oracle_sparse_attention_rows.  These are the
 * numerator and normaliser whose unbiasedness the SIP paragraph states.
 * fp64; nhat [d]. */
void oracle_ht_parts(const uint16_t *q, int d, const uint16_t *k,
                     const uint16_t *v, int64_t N, const int32_t *blocks,
                     const float *log_pi, int count, double scale,
                     double m_ref, double *nhat, double *dhat);

/* Whole-layer drivers over [B,H,N,d] bf16 arrays (OpenMP over (b,h)).
 * Row selection: only query blocks qb with qb_lo <= qb < qb_hi are computed
 * (pass 0 and NQB for all). */
void oracle_select_scores(int B, int H, int64_t N, int d, int nc, int iters,
                          double scale, const uint16_t *q, const uint16_t *k,
                          int qb_lo, int qb_hi, float *scores /*[B,H,NQB,NKB]*/,
                          float *mu /*[B,H,NQB,nc,d]*/, float *w /*[B,H,NQB,nc]*/,
                          int32_t *assign /*[B,H,NQB,128]*/);

/* Plan for every row of a [B,H,NQB,NKB] score array.  kv_index/log_pi are
 * [B,H,NQB,cap]; counts [B,H,NQB] (clipped to cap); r_R [B,H,NQB,2].
 * Returns the number of rows whose sample exceeded cap. */
int oracle_sample_plan(int B, int H, int nqb, int nkb, int64_t n,
                       uint64_t seed, const float *scores, int cap,
                       int32_t *counts, int32_t *kv_index, float *log_pi,
                       uint64_t *r_R);

/* oracle_sample_plan with the design chosen: 0 Poisson, 1 systematic
 * (oracle_sample_row_systematic), 2 paired Poisson.  Paired: the Poisson
 * design whose draws for query block qb are those of query block
 * qb & ~1 of the same (b,h) (counter row ((b*H + h)*NQB + (qb & ~1))), so the
 * two query blocks of a pair share one uniform per KV block.  Each row is
 * still a Poisson sample with its own pi (the Horvitz-Thompson estimate of
 * every row stays unbiased); across a pair, block j is in the sample with the
 * smaller pi_j only if it is in the other (the samples nest block by block),
 * so their union has expected size sum_j max(pi_0j, pi_1j).  A last query
 * block without a partner (NQB odd) keeps its own draws. */
int oracle_sample_plan_design(int B, int H, int nqb, int nkb, int64_t n,
                              uint64_t seed, const float *scores, int cap,
                              int32_t *counts, int32_t *kv_index, float *log_pi,
                              uint64_t *r_R, int design);

/* HT sparse attention for every valid query row of query blocks
 * qb_lo <= qb < qb_hi with the given plan.  o is [B,H,N,d] fp64; rows
 * outside the range are left untouched. */
void oracle_sparse_attention(int B, int H, int64_t N, int d, double scale,
                             const uint16_t *q, const uint16_t *k,
                             const uint16_t *v, int nqb, int cap,
                             const int32_t *counts, const int32_t *kv_index,
                             const float *log_pi, int qb_lo, int qb_hi,
                             double *o);

/* Number of threads the whole-layer drivers use. */
int oracle_num_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* ABSA_ORACLE_H */
