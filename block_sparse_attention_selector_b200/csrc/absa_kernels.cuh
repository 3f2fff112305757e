// absa_kernels.cuh -- host-side launchers of the AB-Attention kernels (sm_100a).
// Each kernel lives in its own translation unit; the C ABI (api.cu) validates
// arguments and calls these.
#pragma once

#include "absa_device.cuh"

namespace absa {

constexpr int kSampleMaxKvBlocks = 49152;

// K1 + K2: per-query-block k-means (8 clusters): centroids, their fp16 split,
// weights and final assignment; the same CTA also writes the mean key of the
// 32 key blocks of its 128-token range as fp16 hi + lo.
cudaError_t launch_kmeans_pool(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int64_t BH, int N,
                               int nqb, int nkb, int d, int iters, float *mu, __half *mu_hi,
                               __half *mu_lo, float *w, uint8_t *assign, __half *kbar_hi,
                               __half *kbar_lo, cudaStream_t stream);

// K3: block scores from the centroids (fp16 hi) and the key-block split (fp16
// hi + lo), in three launches (partial log-sum-exp per key range, combine,
// scores).  part_m/part_s hold [BH, score_key_ranges(nkb), NQB*8] floats, L
// [BH, NQB*8].
int score_key_ranges(int nkb);
cudaError_t launch_score(const CUtensorMap &tm_kb_hi, const CUtensorMap &tm_kb_lo,
                         const CUtensorMap &tm_mu_hi, const float *w, float *part_m,
                         float *part_s, float *L, float *scores, int64_t BH, int nqb, int nkb,
                         int d, float softmax_scale, int32_t *status, cudaStream_t stream);

// K4: SIP plan rows from a score array.  design is an ABSA_SAMPLING_* value;
// nqb (query blocks per head) places each global row in its query-block pair.
cudaError_t launch_sample(const float *scores, int64_t rows, int nkb, int64_t n, uint64_t seed,
                          int design, int nqb, int cap, int32_t *counts, int32_t *kv_index, float *log_pi,
                          uint64_t *r_R, int32_t *status, int64_t row0, cudaStream_t stream);

// Self-test of the bounded device wait: one warp waits on an mbarrier that
// nothing arrives at, with a limit of limit_cycles SM clocks; no copy or MMA
// is in flight.  Sets ABSA_DEVFLAG_TIMEOUT in *status when the wait gives up.
cudaError_t launch_wait_selftest(int32_t *status, long long limit_cycles, cudaStream_t stream);

// K5 (dense = false) / K6 (dense = true): attention of 128-query tiles over
// key tiles of kAttnTileKeys rows.  tq: q as [B*H*N, d] bf16 with a 64 x 128
// box; tk / tv: k / v with a 64 x 4 box (sparse: one 4-token block per box)
// or a 64 x kAttnTileKeys box (dense tiles).
constexpr int kAttnTileKeys = 64;

// Remainder mode of K5 (ESTRA-style): after the plan's tiles, tiles of 64
// group representatives (groups of kRemGroupBlocks consecutive key blocks).
constexpr int kRemGroupBlocks = 32;
constexpr int kRemMaxGroups = (kSampleMaxKvBlocks + kRemGroupBlocks - 1) / kRemGroupBlocks;
struct RemainderArgs {
    CUtensorMap tm_mu, tm_nu;  // group mean keys / values, [B*H*G, d] bf16, 64-row boxes
    const float *gvar;         // [B*H*G] key variance per dimension, averaged over dimensions
    const int32_t *gcnt;       // [B*H*G] tokens per group
    int ngroups;               // G, groups per head
    float var_coef;            // softmax_scale^2 / 2 * log2(e)
};
// K7a: the group statistics of K and V for the remainder mode.
cudaError_t launch_group_stats(const __nv_bfloat16 *k, const __nv_bfloat16 *v, int64_t BH, int N,
                               int d, int ngroups, __nv_bfloat16 *mu, __nv_bfloat16 *nu,
                               float *gvar, int32_t *gcnt, cudaStream_t stream);

// rem != nullptr selects the remainder mode (sparse only).
cudaError_t launch_attention(bool dense, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, const __nv_bfloat16 *k,
                             const __nv_bfloat16 *v, __nv_bfloat16 *o, int64_t BH, int N, int nqb,
                             int nkb, int d, float softmax_scale, const int32_t *counts,
                             const int32_t *kv_index, const float *log_pi, int cap,
                             int32_t *status, cudaStream_t stream,
                             const RemainderArgs *rem = nullptr);

// K5 under the paired design: one CTA per pair of query blocks (2p, 2p+1) of
// a head, gathering the union of the two plan rows once.  The union list is
// held in shared memory, so the host uses it only for 2 * cap <= kPairUnionMax.
constexpr int kPairUnionMax = 6144;
cudaError_t launch_attention_pair(const CUtensorMap &tq, const CUtensorMap &tk,
                                  const CUtensorMap &tv, __nv_bfloat16 *o, int64_t BH, int N,
                                  int nqb, int nkb, int d, float softmax_scale,
                                  const int32_t *counts, const int32_t *kv_index,
                                  const float *log_pi, int cap, int32_t *status,
                                  cudaStream_t stream);

}  // namespace absa
