// score.cu -- IBCS block score on sm_100a (AB-Attention summary page,
// "AB-Attention's three techniques", IBCS paragraph: the weighted attention of
// a block's centroids to every key block's averaged key):
//   s[qb, j] = sum_c w_c * softmax_j(scale * mu_c . kbar_j)   over all key blocks j.
//
// The softmax runs over every key block of the head, so each centroid needs
// its log-sum-exp over all of them before any score can be formed.  The work
// is split by key range instead of by query block: a CTA keeps 256 key blocks
// (two 128-row tiles, fp16 hi + lo) resident in shared memory and streams the
// head's centroid tiles (128 rows = 16 query blocks x 8 clusters, fp16) past
// them, so each key tile is read from memory once per pass instead of once per
// group of query blocks.
//   K3a absa_score_lse_kernel      per (head, key range): for every centroid
//       row, max and sum of exp2 of its logits over the range (partials);
//   K3b absa_score_combine_kernel  per centroid: L = log2-sum-exp over the
//       ranges minus log2(w) (+inf for an empty cluster);
//   K3c absa_score_out_kernel      per (head, key range): the logits again,
//       transposed (thread = key block), s = sum_c exp2(scaled logit - L_c).
// Logits of the score pass are mu_hi . (kbar_hi + kbar_lo) from two fp16
// tcgen05 MMAs per k-step; kbar is carried to about 2^-22 and mu to fp16
// (relative rounding 2^-12 on average), so a workload logit (|l| up to about
// 6 after scaling) is off by about 1e-4 at most, an order below the 1e-3
// score tolerance.  The log-sum-exp pass uses mu_hi . kbar_hi alone (see
// ScoreCta::kLo).
#include "absa_kernels.cuh"

namespace absa {

constexpr int kScoreKeyTiles = 2;                    // key tiles (128 key blocks) per CTA
constexpr int kScoreRange = 128 * kScoreKeyTiles;    // key blocks per CTA
constexpr int kScoreGroupWarps = 8;                  // epilogue warps per group
constexpr int kScoreThreads = 32 * (2 + 2 * kScoreGroupWarps);  // 0 TMA, 1 MMA, 2..17 epilogue

template <int D>
struct Score2Smem {
    static constexpr int kRegions = D / 64;                      // 64-element SW128 regions
    static constexpr int kTile = 128 * 128;                      // one region of 128 rows (bytes)
    static constexpr int kKeyTileBytes = 2 * kRegions * kTile;   // hi + lo of 128 key blocks
    static constexpr int kMuTileBytes = kRegions * kTile;        // 128 centroid rows (hi)
    // key blocks of the range: [hi | lo][region][256 rows] (region r of both
    // key tiles contiguous, so that one MMA can take all 256 rows as N)
    static constexpr int kKeyRegion = kScoreKeyTiles * kTile;    // 256 rows of one region
    static constexpr int kKeyLoOff = kRegions * kKeyRegion;      // lo parts after the hi parts
    static constexpr int kKeyOff = 0;
    static constexpr int kMuOff = kScoreKeyTiles * kKeyTileBytes;  // 2-stage centroid ring
    static constexpr int kXOff = kMuOff + 2 * kMuTileBytes;      // f32 [group][slot][2][128] exchange
    static constexpr int kBarOff = kXOff + 2 * 2 * 2 * 128 * 4;
    static constexpr int kBytes = kBarOff + 16 * 8;
    // one CTA per SM: every CTA holds all 512 TMEM columns
    static constexpr int kAlloc = (kBytes + 1024 > 120 * 1024) ? kBytes + 1024 : 120 * 1024;
};

// Producer/MMA/epilogue skeleton shared by the two passes.  TRANSPOSED = false:
// D[centroid row, key block] = mu_hi . (kbar_hi + kbar_lo) (A = centroid tile,
// B = key tile); true: D[key block, centroid row] = (kbar_hi + kbar_lo) . mu_hi
// (A = key tile, B = centroid tile).  D of centroid tile m sits in TMEM
// buffer m & 1 (256 columns: key tile kt at column 128 kt).
template <int D, bool TRANSPOSED>
struct ScoreCta {
    using S = Score2Smem<D>;
    // The log-sum-exp pass (not transposed) takes the logits mu_hi . kbar_hi
    // alone: the dropped mu_hi . kbar_lo moves a scaled logit by about 1e-4
    // (kbar_lo is the fp16 rounding remainder, 2^-11 of kbar), and the
    // normaliser, a softmax-weighted average of exp over all key blocks,
    // moves by the weighted mean of those shifts, well below the 1e-3 score
    // tolerance.  The score pass needs each logit, so it keeps both products.
    static constexpr bool kLo = TRANSPOSED;
    uint8_t *sm;
    uint64_t *key_full, *mu_full, *mu_empty, *d_full, *d_empty;
    uint32_t *tmem_slot;
    volatile int *abort_flag;

    __device__ explicit ScoreCta(uint8_t *raw) {
        sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                         ~uintptr_t(1023));
        uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBarOff);
        key_full = bars + 0;
        mu_full = bars + 1;   // [2]
        mu_empty = bars + 3;  // [2]
        d_full = bars + 5;    // [2]
        d_empty = bars + 7;   // [2]
        tmem_slot = reinterpret_cast<uint32_t *>(bars + 9);
        abort_flag = reinterpret_cast<volatile int *>(bars + 10);
    }

    __device__ uint32_t setup() {
        const int warp = threadIdx.x >> 5;
        if (threadIdx.x == 0) {
            mbar_init(key_full, 1);
            for (int s = 0; s < 2; ++s) {
                mbar_init(mu_full + s, 1);
                mbar_init(mu_empty + s, 1);
                mbar_init(d_full + s, 1);
                mbar_init(d_empty + s, kScoreGroupWarps);
            }
            *abort_flag = 0;
            mbar_fence_init();
        }
        if (warp == 1) tmem_alloc(tmem_slot, 512);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        return *tmem_slot;
    }

    __device__ void teardown(uint32_t tmem) {
        tc_fence_before();
        __syncthreads();
        if ((threadIdx.x >> 5) == 1) {
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, 512);
        }
    }

    // warp 0, one thread: the key tiles once, then the centroid tiles of the head
    __device__ void produce(const CUtensorMap *tm_kb_hi, const CUtensorMap *tm_kb_lo,
                            const CUtensorMap *tm_mu_hi, int key_row0, int mu_row0, int nmt,
                            int32_t *status) {
        tma_prefetch_desc(tm_mu_hi);
        mbar_arrive_expect_tx(key_full, kScoreKeyTiles * S::kKeyTileBytes / (kLo ? 1 : 2));
        const uint32_t kbase = smem_u32(sm + S::kKeyOff);
        for (int kt = 0; kt < kScoreKeyTiles; ++kt)
            for (int r = 0; r < S::kRegions; ++r) {
                const uint32_t off = r * S::kKeyRegion + kt * S::kTile;
                tma_load_2d(kbase + off, tm_kb_hi, 64 * r, key_row0 + 128 * kt, key_full);
                if (kLo)
                    tma_load_2d(kbase + S::kKeyLoOff + off, tm_kb_lo, 64 * r, key_row0 + 128 * kt,
                                key_full);
            }
        for (int m = 0; m < nmt; ++m) {
            const int st = m & 1;
            if (m >= 2 && !mbar_wait(mu_empty + st, ((m - 2) >> 1) & 1, status, abort_flag, 0))
                break;
            mbar_arrive_expect_tx(mu_full + st, S::kMuTileBytes);
            const uint32_t base = smem_u32(sm + S::kMuOff + st * S::kMuTileBytes);
            for (int r = 0; r < S::kRegions; ++r)
                tma_load_2d(base + r * S::kTile, tm_mu_hi, 64 * r, mu_row0 + 128 * m, mu_full + st);
        }
    }

    // warp 1, one thread
    __device__ void mma(uint32_t tmem, int nmt, int32_t *status) {
        constexpr uint32_t idesc128 = idesc_f16_f32(128, 128, 0);
        constexpr uint32_t idesc256 = idesc_f16_f32(128, 256, 0);
        if (!mbar_wait(key_full, 0, status, abort_flag)) return;
        const uint32_t kbase = smem_u32(sm + S::kKeyOff);
        for (int m = 0; m < nmt; ++m) {
            const int st = m & 1, buf = m & 1;
            if (!mbar_wait(mu_full + st, (m >> 1) & 1, status, abort_flag)) return;
            if (m >= 2 && !mbar_wait(d_empty + buf, ((m - 2) >> 1) & 1, status, abort_flag))
                return;
            tc_fence_after();
            const uint32_t mu_base = smem_u32(sm + S::kMuOff + st * S::kMuTileBytes);
            if (TRANSPOSED) {
                // D[key, centroid] per key tile: A = 128 key rows (hi, then lo), B = centroids
#pragma unroll
                for (int kt = 0; kt < kScoreKeyTiles; ++kt) {
                    const uint32_t dt = tmem + buf * 256 + kt * 128;
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t koff = (ks >> 2) * S::kKeyRegion + kt * S::kTile + (ks & 3) * 32;
                        const uint32_t moff = (ks >> 2) * S::kTile + (ks & 3) * 32;
                        const uint64_t mu_d = sw128_desc(mu_base + moff, 16, 1024);
                        tc_mma_f16(dt, sw128_desc(kbase + koff, 16, 1024), mu_d, idesc128, ks > 0);
                        tc_mma_f16(dt, sw128_desc(kbase + S::kKeyLoOff + koff, 16, 1024), mu_d,
                                   idesc128, 1);
                    }
                }
            } else {
                // D[centroid, key] for all 256 key blocks at once: N = 256
                const uint32_t dt = tmem + buf * 256;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t koff = (ks >> 2) * S::kKeyRegion + (ks & 3) * 32;
                    const uint32_t moff = (ks >> 2) * S::kTile + (ks & 3) * 32;
                    const uint64_t mu_d = sw128_desc(mu_base + moff, 16, 1024);
                    tc_mma_f16(dt, mu_d, sw128_desc(kbase + koff, 16, 1024), idesc256, ks > 0);
                    if (kLo)
                        tc_mma_f16(dt, mu_d, sw128_desc(kbase + S::kKeyLoOff + koff, 16, 1024),
                                   idesc256, 1);
                }
            }
            tc_commit(d_full + buf);
            tc_commit(mu_empty + st);
        }
    }
};

// K3a: partial log-sum-exp of every centroid row over one key range.
// Epilogue warp w: TMEM lane quarter w % 4 (centroid rows), key tile
// (w - 2) / 4; the two key tiles of a row are merged through shared memory.
template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1) absa_score_lse_kernel(
    const __grid_constant__ CUtensorMap tm_kb_hi, const __grid_constant__ CUtensorMap tm_kb_lo,
    const __grid_constant__ CUtensorMap tm_mu_hi, float *__restrict__ part_m,
    float *__restrict__ part_s, int nqb, int nkb, int nkr, float scale_log2, int32_t *status) {
    using S = Score2Smem<D>;
    extern __shared__ uint8_t score2_smem_raw[];
    ScoreCta<D, false> cta(score2_smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = blockIdx.x / nkr;
    const int kr = blockIdx.x % nkr;
    const int nrows = nqb * 8, nmt = (nrows + 127) / 128;
    const uint32_t tmem = cta.setup();

    if (warp == 0) {
        if (lane == 0)
            cta.produce(&tm_kb_hi, &tm_kb_lo, &tm_mu_hi, (int)(bh * nkb + kr * kScoreRange),
                        (int)(bh * nrows), nmt, status);
    } else if (warp == 1) {
        if (lane == 0) cta.mma(tmem, nmt, status);
    } else {
        // epilogue group g takes the centroid tiles m = g, g + 2, ... (TMEM
        // buffer g), so one group's exponentials overlap the other's loads,
        // maxima and exchange; within a group, warp w: TMEM lane quarter
        // w % 4, key tile (w % 8) / 4
        const int e = warp - 2, g = e / kScoreGroupWarps, we = e % kScoreGroupWarps;
        const int quarter = warp & 3, half = we >> 2;
        const int r = quarter * 32 + lane;
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + half * 128;
        const int ncols = min(128, nkb - kr * kScoreRange - half * 128);  // valid key blocks
        float *xch = reinterpret_cast<float *>(cta.sm + S::kXOff);  // [g][slot][max|sum][row]
        // every warp of a group passes the group's named barrier once per tile
        // of the group, also after a failed wait (then without touching TMEM)
        bool ok = true;
        for (int m = g; m < nmt; m += 2) {
            const int buf = g;
            if (ok)
                ok = __all_sync(0xffffffffu,
                                mbar_wait(cta.d_full + buf, (m >> 1) & 1, status, cta.abort_flag));
            if (ok) tc_fence_after();
            float mx = -INFINITY, sum = 0.f;
#pragma unroll 1
            for (int ch = 0; ch < 2 && ok; ++ch) {  // 64 columns at a time
                uint32_t v[2][32];
                tmem_ld32(lane_addr + buf * 256 + ch * 64, v[0]);
                tmem_ld32(lane_addr + buf * 256 + ch * 64 + 32, v[1]);
                tmem_wait_ld();
                if (ch == 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(cta.d_empty + buf);
                }
                const int nc = min(64, ncols - ch * 64);
                if (nc <= 0) continue;
                if (nc < 64) {  // the last key blocks of the head: mask the rest with -inf
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (i >= nc) v[i >> 5][i & 31] = __float_as_uint(-INFINITY);
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(v[i >> 5][i & 31]));
                const float cmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                if (cmax > mx) {
                    sum *= ex2((mx - cmax) * scale_log2);
                    mx = cmax;
                }
                const float moff = -mx * scale_log2;
                float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 64; ++i)  // exp2(-inf) = 0 for the masked columns
                    a4[i & 3] += ex2(__fmaf_rn(__uint_as_float(v[i >> 5][i & 31]), scale_log2, moff));
                sum += (a4[0] + a4[1]) + (a4[2] + a4[3]);
            }
            // two exchange slots per group, alternating with the group's tiles:
            // a slot is rewritten two group tiles later, after the group's
            // barrier of the tile in between
            float *x = xch + (g * 2 + ((m >> 1) & 1)) * 256;
            if (half == 1) {
                x[r] = mx;
                x[128 + r] = sum;
            }
            asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");
            if (half == 0 && ok) {
                const float m1 = x[r], s1 = x[128 + r];
                const float mm = fmaxf(mx, m1);
                const float tot = (mx == -INFINITY ? 0.f : sum * ex2((mx - mm) * scale_log2)) +
                                  (m1 == -INFINITY ? 0.f : s1 * ex2((m1 - mm) * scale_log2));
                const int crow = m * 128 + r;
                if (crow < nrows) {
                    const int64_t o = (bh * nkr + kr) * (int64_t)nrows + crow;
                    part_m[o] = mm;
                    part_s[o] = tot;
                }
            }
        }
    }
    cta.teardown(tmem);
}

// K3b: L_c = log2(sum over key ranges of sum_j exp2(scaled logit)) - log2(w_c).
__global__ void __launch_bounds__(256) absa_score_combine_kernel(
    const float *__restrict__ part_m, const float *__restrict__ part_s, const float *__restrict__ w,
    float *__restrict__ L, int nrows, int nkr, int64_t total_rows, float scale_log2) {
    const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= total_rows) return;
    const int64_t bh = i / nrows;
    const int crow = (int)(i % nrows);
    const float *pm = part_m + bh * nkr * (int64_t)nrows + crow;
    const float *ps = part_s + bh * nkr * (int64_t)nrows + crow;
    float mm = -INFINITY;
    for (int k = 0; k < nkr; ++k) mm = fmaxf(mm, pm[(int64_t)k * nrows]);
    float tot = 0.f;
    for (int k = 0; k < nkr; ++k) {
        const float mk = pm[(int64_t)k * nrows];
        if (mk != -INFINITY) tot += ps[(int64_t)k * nrows] * ex2((mk - mm) * scale_log2);
    }
    const float wc = w[i];
    L[i] = wc > 0.f ? mm * scale_log2 + log2f(tot) - log2f(wc) : INFINITY;
}

// K3c: scores of every query block for the key blocks of one key range.
// Epilogue warp w: TMEM lane quarter w % 4 (key blocks of key tile
// (w - 2) / 4); a thread forms, for each query block of a centroid tile,
// s_j = sum over its 8 centroids of exp2(scaled logit - L_c).
template <int D>
__global__ void __launch_bounds__(kScoreThreads, 1) absa_score_out_kernel(
    const __grid_constant__ CUtensorMap tm_kb_hi, const __grid_constant__ CUtensorMap tm_kb_lo,
    const __grid_constant__ CUtensorMap tm_mu_hi, const float *__restrict__ L,
    float *__restrict__ scores, int nqb, int nkb, int nkr, float scale_log2, int32_t *status) {
    extern __shared__ uint8_t score2_smem_raw[];
    ScoreCta<D, true> cta(score2_smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t bh = blockIdx.x / nkr;
    const int kr = blockIdx.x % nkr;
    const int nrows = nqb * 8, nmt = (nrows + 127) / 128;
    const uint32_t tmem = cta.setup();

    if (warp == 0) {
        if (lane == 0)
            cta.produce(&tm_kb_hi, &tm_kb_lo, &tm_mu_hi, (int)(bh * nkb + kr * kScoreRange),
                        (int)(bh * nrows), nmt, status);
    } else if (warp == 1) {
        if (lane == 0) cta.mma(tmem, nmt, status);
    } else {
        // epilogue group g takes the centroid tiles m = g, g + 2, ... (TMEM
        // buffer g); within a group, warp w: TMEM lane quarter w % 4 (key
        // blocks), key tile (w % 8) / 4
        const int e8 = warp - 2, g = e8 / kScoreGroupWarps, we = e8 % kScoreGroupWarps;
        const int quarter = warp & 3, half = we >> 2;
        const int j = kr * kScoreRange + half * 128 + quarter * 32 + lane;  // key block
        const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16) + half * 128;
        const float *Lh = L + bh * (int64_t)nrows;
        float *sh = scores + bh * (int64_t)nqb * nkb;
        // L of the group's centroid tile in shared memory (two slots per group,
        // alternating with its tiles); group thread e < 128 fetches row e of
        // the group's next tile while the current one is processed
        float *Lg = reinterpret_cast<float *>(cta.sm + Score2Smem<D>::kXOff) + g * 256;
        const int e = we * 32 + lane;
        float lnext = (g * 128 + e < nrows && g < nmt) ? __ldg(Lh + g * 128 + e) : INFINITY;
        bool ok = true;
        for (int m = g; m < nmt; m += 2) {
            const int buf = g;
            float *Ls = Lg + ((m >> 1) & 1) * 128;
            if (e < 128) Ls[e] = lnext;
            asm volatile("bar.sync %0, 256;" ::"r"(1 + g) : "memory");  // every warp, every tile
            if (e < 128 && m + 2 < nmt) {
                const int row = (m + 2) * 128 + e;
                lnext = row < nrows ? __ldg(Lh + row) : INFINITY;
            }
            if (ok)
                ok = __all_sync(0xffffffffu,
                                mbar_wait(cta.d_full + buf, (m >> 1) & 1, status, cta.abort_flag));
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int ch = 0; ch < 2; ++ch) {  // 64 centroid columns = 8 query blocks
                    uint32_t v[2][32];
                    tmem_ld32(lane_addr + buf * 256 + ch * 64, v[0]);
                    tmem_ld32(lane_addr + buf * 256 + ch * 64 + 32, v[1]);
                    tmem_wait_ld();
                    if (ch == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(cta.d_empty + buf);
                    }
                    if (j >= nkb) continue;
#pragma unroll
                    for (int qbl = 0; qbl < 8; ++qbl) {
                        const int qb = m * 16 + ch * 8 + qbl;
                        if (qb >= nqb) break;
                        const float4 L0 = *reinterpret_cast<const float4 *>(Ls + (ch * 8 + qbl) * 8);
                        const float4 L1 = *reinterpret_cast<const float4 *>(Ls + (ch * 8 + qbl) * 8 + 4);
                        const float Lc[8] = {L0.x, L0.y, L0.z, L0.w, L1.x, L1.y, L1.z, L1.w};
                        float s2[2] = {0.f, 0.f};
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int col = qbl * 8 + c;
                            s2[c & 1] += ex2(__fmaf_rn(__uint_as_float(v[col >> 5][col & 31]),
                                                       scale_log2, -Lc[c]));
                        }
                        sh[(int64_t)qb * nkb + j] = s2[0] + s2[1];
                    }
                }
            }
        }
    }
    cta.teardown(tmem);
}

template <int D>
static cudaError_t launch_score_d(const CUtensorMap &kb_hi, const CUtensorMap &kb_lo,
                                  const CUtensorMap &mu_hi, const float *w, float *part_m,
                                  float *part_s, float *L, float *scores, int64_t BH, int nqb,
                                  int nkb, float scale_log2, int32_t *status,
                                  cudaStream_t stream) {
    const int smem = Score2Smem<D>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(absa_score_lse_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(absa_score_out_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int nkr = (nkb + kScoreRange - 1) / kScoreRange;
    const unsigned grid = (unsigned)(BH * nkr);
    absa_score_lse_kernel<D><<<grid, kScoreThreads, smem, stream>>>(
        kb_hi, kb_lo, mu_hi, part_m, part_s, nqb, nkb, nkr, scale_log2, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t rows = BH * nqb * 8;
    absa_score_combine_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(
        part_m, part_s, w, L, nqb * 8, nkr, rows, scale_log2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    absa_score_out_kernel<D><<<grid, kScoreThreads, smem, stream>>>(
        kb_hi, kb_lo, mu_hi, L, scores, nqb, nkb, nkr, scale_log2, status);
    return cudaGetLastError();
}

int score_key_ranges(int nkb) { return (nkb + kScoreRange - 1) / kScoreRange; }

cudaError_t launch_score(const CUtensorMap &tm_kb_hi, const CUtensorMap &tm_kb_lo,
                         const CUtensorMap &tm_mu_hi, const float *w, float *part_m,
                         float *part_s, float *L, float *scores, int64_t BH, int nqb, int nkb,
                         int d, float softmax_scale, int32_t *status, cudaStream_t stream) {
    const float scale_log2 = softmax_scale * 1.4426950408889634f;
    return d == 64 ? launch_score_d<64>(tm_kb_hi, tm_kb_lo, tm_mu_hi, w, part_m, part_s, L,
                                        scores, BH, nqb, nkb, scale_log2, status, stream)
                   : launch_score_d<128>(tm_kb_hi, tm_kb_lo, tm_mu_hi, w, part_m, part_s, L,
                                         scores, BH, nqb, nkb, scale_log2, status, stream);
}

}  // namespace absa
