/*
 * absa.h -- C ABI of the B200 (sm_100a) AB-Attention hot path:
 * IBCS block selector, SIP sampler and Horvitz-Thompson sparse attention
 * over 4-token key/value blocks, plus a dense attention kernel for
 * comparison.
 *
 * Method source: "AB-Attention speeds up video generation by up to 2.23x and
 * skips 92% of attention" (news.hamidun.com), section "AB-Attention's three
 * techniques" -- IBCS paragraph (selector), SIP paragraph (sampler and 1/pi
 * logit shift), third paragraph (4-token blocks gathered into full tensor-core
 * tiles, plan reused for four denoising steps); and the HF daily-papers
 * summary (zerohour.day) "Key facts": no token permutation, sub-tile blocks
 * packed into full tensor-core tiles.
 *
 * Conventions shared by every entry point
 *  - Tensors are caller-owned DEVICE memory; q, k, v, o are bf16 [B,H,N,d]
 *    row-major (d fastest).  Token n of a T x Hg x Wg latent grid is
 *    n = (t*Hg + y)*Wg + x and is never permuted.
 *  - Query block qb holds tokens 128*qb .. min(128*qb+127, N-1)
 *    (NQB = ceil(N/128)); key/value block j holds tokens 4j .. min(4j+3, N-1)
 *    (NKB = ceil(N/4)).
 *  - Work is enqueued on `stream` (a cudaStream_t; 0 = legacy default).  The
 *    library never allocates, frees or synchronises, except absa_plan_check
 *    and absa_select_check, which synchronise the stream to read a device
 *    status word.  Every entry point opens an NVTX range of its own name.
 *  - Pointers must be 16-byte aligned.  Host-detectable errors return before
 *    any launch; launch failures return ABSA_ERR_CUDA; errors seen on the
 *    device are OR-ed into a device status word (ABSA_DEVFLAG_*).
 *  - No CPU fallback: unsupported shapes return ABSA_ERR_UNSUPPORTED.
 *  - Inputs are never written.
 */
#ifndef ABSA_H
#define ABSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ABSA_OK = 0,
    ABSA_ERR_INVALID_ARG = 1,   /* bad pointer, alignment, size or field        */
    ABSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (d, block sizes)   */
    ABSA_ERR_WORKSPACE = 3,     /* workspace smaller than absa_workspace_bytes  */
    ABSA_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed         */
    ABSA_ERR_PLAN_OVERFLOW = 5, /* a sample exceeded the plan capacity          */
    ABSA_ERR_BAD_PLAN = 6,      /* plan count/index out of range (seen on GPU)  */
    ABSA_ERR_TIMEOUT = 7        /* a bounded device wait ran out                */
} absa_status;

/* Bits of the device status word (plan->status / the status argument). */
#define ABSA_DEVFLAG_OVERFLOW 1
#define ABSA_DEVFLAG_BAD_PLAN 2
#define ABSA_DEVFLAG_TIMEOUT 4

typedef struct {
    int32_t B, H, N, d;     /* batch, heads, tokens (= T*Hg*Wg), head dim (64|128)   */
    int32_t T, Hg, Wg;      /* latent grid; token n = (t*Hg + y)*Wg + x               */
    int32_t q_block;        /* must be 128 (IBCS paragraph: blocks of 128 queries)    */
    int32_t kv_block;       /* must be 4 (third paragraph: 4-token KV blocks)         */
    int32_t n_clusters;     /* must be 8 (IBCS paragraph: 8 clusters per block)       */
    int32_t kmeans_iters;   /* Lloyd rounds, 1..16 (3 in every workload)              */
    int32_t budget_blocks;  /* n: expected KV blocks per query block; n >= NKB = dense */
    uint64_t seed;          /* SIP draw seed                                          */
    float softmax_scale;    /* logit scale, normally 1/sqrt(d)                        */
    int32_t sampling;       /* SIP design: ABSA_SAMPLING_POISSON (0, the default),    */
                            /* ABSA_SAMPLING_SYSTEMATIC (1) or ABSA_SAMPLING_PAIRED   */
                            /* (2); see absa_sample_plan                              */
} absa_params;

/* Sampling designs of the SIP sampler (absa_params.sampling). */
#define ABSA_SAMPLING_POISSON 0
#define ABSA_SAMPLING_SYSTEMATIC 1
#define ABSA_SAMPLING_PAIRED 2

typedef struct {
    /* All arrays are caller-owned device memory sized from absa_plan_capacity. */
    int32_t n_qblocks;      /* NQB                                                   */
    int32_t n_kvblocks;     /* NKB                                                   */
    int32_t capacity;       /* entries per row (>= absa_plan_capacity)               */
    int32_t *counts;        /* [B,H,NQB] taken blocks per row (clipped to capacity)  */
    int32_t *kv_index;      /* [B,H,NQB,capacity] ascending block ids, valid to count */
    float *log_pi;          /* [B,H,NQB,capacity] ln(pi) of each entry (0 if pi = 1)  */
    uint64_t *r_R;          /* [B,H,NQB,2] audit: r*, R* of the integer pi solve      */
    int32_t *status;        /* one device word, OR of ABSA_DEVFLAG_*                  */
} absa_plan;

/* Library version string. */
const char *absa_version(void);

/* Human-readable name of a status code (static storage). */
const char *absa_status_string(absa_status s);

/* Validate a parameter block (host only).  Returns ABSA_OK, INVALID_ARG or
 * UNSUPPORTED. */
absa_status absa_check_params(const absa_params *p);

/* Plan row capacity for p: min(NKB, roundup32(n + ceil(8*sqrt(n)) + 32)),
 * i.e. the budget plus eight standard deviations of a Poisson sample size
 * (SIP paragraph: blocks are drawn, so the sample size varies).  Returns -1
 * if p is invalid. */
int32_t absa_plan_capacity(const absa_params *p);

/* Bytes of workspace absa_select_scores / absa_select_plan need.  Layout,
 * each region starting at a 256-byte boundary in this order:
 *   kbar_hi  fp16 [B,H,NKB,d]   mean key of every 4-token block, high part
 *   kbar_lo  fp16 [B,H,NKB,d]   low part (kbar ~= hi + lo to about 2^-22)
 *   mu       f32  [B,H,NQB,8,d] final k-means centroids
 *   mu_hi    fp16 [B,H,NQB,8,d] fp16(mu), the centroid operand of the score
 *   mu_lo    fp16 [B,H,NQB,8,d] fp16(mu - mu_hi) (audit only)
 *   w        f32  [B,H,NQB,8]   centroid weights |c| / n_valid
 *   assign   u8   [B,H,NQB,128] final assignment (255 for padded rows)
 *   part_m   f32  [B,H,NKR,NQB*8] per key range of 256 key blocks
 *                               (NKR = ceil(NKB/256)) and centroid row: the
 *                               largest logit mu . kbar over the range
 *   part_s   f32  [B,H,NKR,NQB*8] sum over the range of exp of the scaled
 *                               logit minus that largest one (base 2)
 *   lse      f32  [B,H,NQB*8]   L = log2-sum-exp of the scaled logits over
 *                               all key blocks minus log2(w) (+inf if w = 0)
 *   status   i32  [1]           device status word of the score stage
 *                               (ABSA_DEVFLAG_TIMEOUT); read it with
 *                               absa_select_check
 * The regions after kbar_lo are readable audit outputs of the last call.
 * Returns 0 if p is invalid. */
size_t absa_workspace_bytes(const absa_params *p);

/* IBCS selector (IBCS paragraph): for every (b,h) pool the keys of each
 * 4-token block into their mean, run the per-128-query-block k-means
 * (8 clusters, kmeans_iters Lloyd rounds in fp32, initial centroids the
 * queries at offsets floor(c*m/8), ties to the lowest index, empty clusters
 * keep their centroid), weight each centroid by its share of the block's m
 * valid queries, and write
 *   scores[b,h,qb,j] = sum_c w_c * softmax_j(softmax_scale * mu_c . kbar_j)
 * (f32 [B,H,NQB,NKB], each row sums to 1).  The products mu_c . kbar_j run
 * on the tensor cores as fp16(mu_c) . (kbar_hi + kbar_lo); inputs whose
 * magnitude exceeds the fp16 range (65504) are clamped to it, which only
 * the accuracy of the scores can notice.  ws must hold
 * absa_workspace_bytes(p) bytes (ABSA_ERR_WORKSPACE otherwise).  The call
 * resets the workspace's status word first; a bounded wait of the score
 * kernels that runs out sets ABSA_DEVFLAG_TIMEOUT there (the scores are then
 * incomplete), which absa_select_check reports.  Equivalent to
 * absa_select_pool_kmeans followed by absa_select_block_scores on the same
 * workspace. */
absa_status absa_select_scores(const absa_params *p, const void *q, const void *k,
                               float *scores, void *ws, size_t ws_bytes, void *stream);

/* First half of absa_select_scores (IBCS paragraph: "averaged keys" and the
 * per-block k-means): writes the kbar_hi/kbar_lo, mu, mu_hi, mu_lo, w and
 * assign regions of ws.  The k-means kernel has no device waits and does not
 * touch the status word.  Arguments and errors as absa_select_scores. */
absa_status absa_select_pool_kmeans(const absa_params *p, const void *q, const void *k, void *ws,
                                    size_t ws_bytes, void *stream);

/* Second half of absa_select_scores (IBCS paragraph: weighted centroid
 * attention to the averaged keys): the scores from the regions written by
 * absa_select_pool_kmeans on the same ws (and the same p).  Resets the
 * workspace's status word first.  Arguments and errors as
 * absa_select_scores. */
absa_status absa_select_block_scores(const absa_params *p, float *scores, void *ws,
                                     size_t ws_bytes, void *stream);

/* Synchronise `stream` and read the selector's status word: the one in ws
 * (the workspace of absa_select_scores / absa_select_block_scores), or, with
 * ws = NULL, the one in the built-in array of absa_select_scores_static on
 * the current device.  Returns ABSA_ERR_TIMEOUT if the last score stage gave
 * up a bounded wait, else ABSA_OK (also INVALID_ARG / WORKSPACE / CUDA for
 * bad arguments or a failing CUDA call).  Does not clear the word.
 * (absa_select_plan and absa_step_host report into plan->status instead.) */
absa_status absa_select_check(const absa_params *p, const void *ws, void *stream);

/* SIP sampler (SIP paragraph) on a score array [B,H,NQB,NKB] f32.
 * Integer inclusion probabilities: q_j = max(1, floor(s_j * 2^32)) (NaN or
 * negative -> 1, at most 2^32); from C = {} repeat r = n - |C|,
 * R = sum_{j not in C} q_j, C += {j : r*q_j >= R} until C is unchanged;
 * pi_j = 1 on C, r*q_j/R elsewhere, so sum pi = n exactly.  Draws: with
 * ctr = row*NKB + j, row = (b*H + h)*NQB + qb, and mix the SplitMix64 output
 * function, u(ctr) = mix(mix(seed) + (ctr+1)*0x9E3779B97F4A7C15) >> 32
 * (output ctr+1 of SplitMix64 started from state mix(seed)).
 *  - ABSA_SAMPLING_POISSON: block j is taken iff j in C or
 *    u(row*NKB + j) * R < r*q_j * 2^32 (independent draws; the sample size
 *    is random with mean n).
 *  - ABSA_SAMPLING_SYSTEMATIC: the blocks are laid end to end in ascending j
 *    with lengths a_j = R on C and r*q_j elsewhere (sum n*R); with
 *    U = u(row*NKB), points sit at (k + U/2^32)*R for k = 0..n-1 and block j
 *    is taken iff a point falls in [sum_{i<j} a_i, sum_{i<=j} a_i).  Every
 *    block is taken with probability pi_j and exactly n blocks are taken.
 *  - ABSA_SAMPLING_PAIRED: the Poisson rule with the draws of query block
 *    qb & ~1 of the same (b,h): block j of row (b,h,qb) is taken iff j in C
 *    or u(row'*NKB + j) * R < r*q_j * 2^32, row' = (b*H + h)*NQB + (qb & ~1).
 *    Each row is still a Poisson sample with its own pi; the two rows of a
 *    pair share one uniform per block, so the row with the smaller pi_j
 *    takes j only if the other does (their samples nest block by block and
 *    their union has expected size sum_j max(pi_0j, pi_1j)).  A last query
 *    block without a partner (NQB odd) keeps its own draws.
 * Taken blocks are written ascending
 * with log_pi = 0 (capped) or (float)ln((double)(r*q_j)/R).  n >= NKB takes
 * every block.  Resets plan->status first; a row with more than
 * plan->capacity blocks keeps the first `capacity` and sets
 * ABSA_DEVFLAG_OVERFLOW.  Requires NKB <= 49152. */
absa_status absa_sample_plan(const absa_params *p, const float *scores, const absa_plan *plan,
                             void *stream);

/* absa_select_scores followed by absa_sample_plan (one plan per call; the
 * third paragraph's schedule recomputes it every fourth denoising step and
 * reuses it in between). */
absa_status absa_select_plan(const absa_params *p, const void *q, const void *k, float *scores,
                             const absa_plan *plan, void *ws, size_t ws_bytes, void *stream);

/* Horvitz-Thompson sparse attention (SIP paragraph; third paragraph): for
 * every valid query i of block qb, over the tokens t of the plan's blocks in
 * ascending order, l_t = softmax_scale * q_i . k_t - log_pi(block of t) and
 * o_i = sum_t softmax(l)_t v_t; an empty plan row gives o_i = 0.  The
 * selected 4-token blocks are gathered by index into 128-token tensor-core
 * tiles (tcgen05, bf16 operands, f32 accumulation); tokens are not
 * permuted.  The plan may come from an earlier step (plan reuse).  Plan
 * counts above capacity or indices outside [0, NKB) are rejected on the
 * device (ABSA_DEVFLAG_BAD_PLAN, the row is written as zeros). */
absa_status absa_sparse_attention(const absa_params *p, const void *q, const void *k,
                                  const void *v, const absa_plan *plan, void *o, void *stream);

/* absa_sparse_attention computed with one CTA per pair of query blocks
 * (2p, 2p+1) of a head (SIP paragraph, with the paired design of
 * absa_sample_plan): the CTA gathers each key/value block of the union of the
 * two plan rows once and runs one softmax chain per query block over it, a
 * block absent from a row entering that row's chain with logit bias -inf.
 * Any plan is accepted (rows out of order or with repeated ids are processed
 * as the concatenation of the two rows), and every row's output is the
 * absa_sparse_attention output up to summation order; bad rows are rejected
 * as there.  The union list lives in shared memory: plan->capacity must be
 * at most 3072 (ABSA_ERR_UNSUPPORTED otherwise).  The paired design makes
 * the union only 10-18% larger than one row, yet on B200 this form measured
 * slower than absa_sparse_attention (two independent single-block CTAs per
 * SM), which the other entry points use; it is kept as the pair-union
 * variant of the attention. */
absa_status absa_sparse_attention_pairs(const absa_params *p, const void *q, const void *k,
                                        const void *v, const absa_plan *plan, void *o,
                                        void *stream);

/* Bytes of workspace absa_remainder_attention needs (0 if p is invalid).
 * With G = ceil(NKB / 32) groups per head, each region at a 256-byte
 * boundary in this order:
 *   mu    bf16 [B,H,G,d]  mean key of each group's tokens
 *   nu    bf16 [B,H,G,d]  mean value
 *   var   f32  [B,H,G]    key variance per dimension, averaged over d
 *   count i32  [B,H,G]    tokens in the group (128, fewer in a head's last) */
size_t absa_remainder_workspace_bytes(const absa_params *p);

/* ESTRA-style attention (ESTRA page, summary and figure: the selected pairs
 * exact, the rest from group averages with a variance-calibrated correction
 * of the representatives' weights), on the plan of this library.  For every
 * valid query i of block qb, one softmax runs over
 *   - the tokens t of the plan row's blocks, logit s q_i.k_t (no ln pi shift:
 *     the plan's blocks are the exact part), and
 *   - one representative per group g of 32 consecutive key blocks (128
 *     tokens), key mu_g and value nu_g (the group's mean key and value),
 *     logit s q_i.mu_g + s^2 |q_i|^2 var_g / 2 + ln(m_g), where m_g is the
 *     number of the group's tokens outside the plan row (no representative if
 *     m_g = 0) and var_g the group's key variance per dimension averaged over
 *     dimensions (the Gaussian moment identity E exp(X) = exp(E X + Var X / 2)
 *     with an isotropic key spread),
 * with s = softmax_scale.  The group statistics are written to ws first
 * (ws_bytes >= absa_remainder_workspace_bytes(p), ABSA_ERR_WORKSPACE
 * otherwise), then the attention kernel runs the plan's tiles followed by
 * ceil(G / 64) tiles of representatives in the same softmax.  Plan checks,
 * bad rows and status as absa_sparse_attention; repeated plan entries are
 * counted as often as they appear. */
absa_status absa_remainder_attention(const absa_params *p, const void *q, const void *k,
                                     const void *v, const absa_plan *plan, void *o, void *ws,
                                     size_t ws_bytes, void *stream);

/* Dense softmax attention (the full-attention reference of the pages'
 * evaluation) with the same tile machinery over contiguous keys.  status is
 * a device word for ABSA_DEVFLAG_TIMEOUT (may be NULL). */
absa_status absa_dense_reference(const absa_params *p, const void *q, const void *k,
                                 const void *v, void *o, int32_t *status, void *stream);

/* Size of the library's built-in scratch array used by
 * absa_select_scores_static (bytes). */
#define ABSA_STATIC_SCRATCH_BYTES ((size_t)64 << 20)

/* Allocation-free variant of absa_select_scores (no counterpart on the
 * pages: a library-interface addition).  It computes exactly what
 * absa_select_scores computes, but takes its workspace from a 64 MiB array
 * compiled into the library instead of a caller buffer, so callers that have
 * no way to obtain device memory beyond their own inputs and outputs can
 * still run the selector: plugin hosts that hand a plugin only its tensors,
 * or code that runs under a memory manager it cannot call into.  The call
 * itself never allocates or frees device memory.
 *  - Limit: p must need at most ABSA_STATIC_SCRATCH_BYTES of workspace
 *    (absa_workspace_bytes(p)); larger problems return ABSA_ERR_WORKSPACE
 *    before any work is enqueued.
 *  - The array exists once per GPU for as long as the library is loaded in
 *    the process; the first call on a device looks up its device address
 *    (with that device current), so make that first call before any stream
 *    capture.  The address is kept for the life of the process: after
 *    cudaDeviceReset on a device it is stale, and this entry point must not
 *    be called on that device again.
 *  - The array ends with the same status word as a caller workspace (reset
 *    by every call); absa_select_check(p, NULL, stream) reads it.
 *  - Every call on a device shares the same array and leaves its contents
 *    behind; nothing in it has to start at zero (each call writes every
 *    region before reading it).  Calls that can run at the same time on one
 *    GPU (different streams, or different host threads) race on the array:
 *    serialise them.
 * Arguments, layout and other errors as absa_select_scores. */
absa_status absa_select_scores_static(const absa_params *p, const void *q, const void *k,
                                      float *scores, void *stream);

/* One whole step on host tensors, pipelined over runs of heads (no
 * counterpart on the pages: a library-interface addition for callers whose
 * q, k, v live in host memory).  For each run of heads_per_run flattened
 * (b,h) heads: copy its q, k, v rows from q_host/k_host/v_host (bf16
 * [B,H,N,d], same layout as on the device) into q/k/v on copy_in_stream,
 * then on `stream` run the selector, the sampler and the sparse attention for
 * those heads, then copy its o rows back into o_host on copy_out_stream.  The
 * copies of one run overlap the compute of the others.  Heads are
 * independent in every stage and the draw counter uses the global plan row,
 * so scores, plan and o equal those of absa_select_plan followed by
 * absa_sparse_attention on the whole problem, for any heads_per_run >= 1.
 *  - q, k, v, o, scores, plan, ws: device buffers as in those calls (caller
 *    owned; q/k/v are overwritten with the host inputs).  ws must hold
 *    absa_workspace_bytes(p) bytes.
 *  - Host buffers must stay valid until the step completes; page-locked host
 *    memory (cudaHostAlloc / cudaHostRegister) is needed for the copies to
 *    overlap, pageable memory gives the same results without overlap.
 *  - copy_in_stream / copy_out_stream may be NULL (then `stream` does the
 *    copies, with no overlap).  Copies into q/k/v wait for the work enqueued
 *    on `stream` before the call; `stream` completes after the last output
 *    copy, so synchronising `stream` makes o_host readable.
 *  - Resets plan->status first.  Creates two CUDA events per run and
 *    destroys them before returning (no device memory is allocated).
 *  - Host-detectable errors return before anything is enqueued; a failing
 *    CUDA call returns ABSA_ERR_CUDA with the earlier runs enqueued. */
absa_status absa_step_host(const absa_params *p, const void *q_host, const void *k_host,
                           const void *v_host, void *o_host, void *q, void *k, void *v, void *o,
                           float *scores, const absa_plan *plan, void *ws, size_t ws_bytes,
                           int32_t heads_per_run, void *stream, void *copy_in_stream,
                           void *copy_out_stream);

/* Self-test of the library's bounded device waits (no counterpart on the
 * pages; it exists so that the timeout path can be exercised without any
 * fault): launches one warp that waits on a shared-memory barrier nothing
 * ever completes, with no copy or MMA in flight, gives up after about
 * limit_cycles SM clocks (1 .. 2e9) and ORs ABSA_DEVFLAG_TIMEOUT into the
 * device word *status.  The kernel then returns normally and the context
 * stays usable. */
absa_status absa_selftest_wait_timeout(int32_t *status, int64_t limit_cycles, void *stream);

/* Synchronise `stream`, read plan->status and map it to a status code
 * (TIMEOUT > BAD_PLAN > OVERFLOW > OK).  Does not clear the word. */
absa_status absa_plan_check(const absa_plan *plan, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ABSA_H */
