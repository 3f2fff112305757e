// sample.cu -- SIP sampler on sm_100a (AB-Attention summary page, "AB-Attention's
// three techniques", SIP paragraph): inclusion probability proportional to the
// block score, the top blocks capped at pi = 1, the rest keeping a nonzero
// chance, sum pi = budget; independent (Poisson) draws from a counter-based
// hash; ascending compaction of the taken blocks with their ln(pi).
//
// Integer formulation (exact, so every ordering of the reductions gives the
// same plan): q_j = max(1, floor(s_j 2^32)); capping fixed point on
// (r, R) = (n - |C|, sum_{j not in C} q_j) with u64 block reductions; draw
// u_j * R < (r q_j) 2^32 compared in 128 bits.
#include "absa_kernels.cuh"

namespace absa {

__device__ __forceinline__ uint64_t quantise_score(float s) {
    const float x = s * 4294967296.0f;  // exact power-of-two scaling
    if (!(x >= 1.0f)) return 1ull;      // NaN, negative, or below one unit
    if (x >= 4294967296.0f) return 1ull << 32;
    return (uint64_t)x;                 // floor for x >= 1
}

__device__ __forceinline__ uint32_t draw_u32(uint64_t seed, uint64_t ctr) {
    uint64_t z = splitmix64_mix(ctr + 0x9E3779B97F4A7C15ull);
    z = splitmix64_mix(z ^ seed);
    return (uint32_t)(z >> 32);
}

// u * R < rq * 2^32 in 128-bit arithmetic (u < 2^32, R and rq < 2^48).
__device__ __forceinline__ bool draw_taken(uint32_t u, uint64_t R, uint64_t rq) {
    const uint64_t lhs_lo = (uint64_t)u * R;
    const uint64_t lhs_hi = __umul64hi((uint64_t)u, R);
    const uint64_t rhs_lo = rq << 32;
    const uint64_t rhs_hi = rq >> 32;
    return lhs_hi < rhs_hi || (lhs_hi == rhs_hi && lhs_lo < rhs_lo);
}

constexpr int kSampleThreads = 512;
constexpr int kSampleWarps = kSampleThreads / 32;

// Block-wide sum of a u64 and an int; result broadcast to every thread.
__device__ __forceinline__ void block_sum2(uint64_t &a, int &b, uint64_t *red_a, int *red_b) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    __syncthreads();  // previous readers of red_* are done
    if (lane == 0) {
        red_a[warp] = a;
        red_b[warp] = b;
    }
    __syncthreads();
    a = 0;
    b = 0;
#pragma unroll
    for (int w = 0; w < kSampleWarps; ++w) {
        a += red_a[w];
        b += red_b[w];
    }
}

// One CTA per plan row (b,h,qb).  The score row is staged in shared memory
// (4 bytes per key block) with one capped flag byte per block.
__global__ void __launch_bounds__(kSampleThreads) absa_sample_kernel(
    const float *__restrict__ scores, int nkb, int64_t n, uint64_t seed, int cap,
    int32_t *__restrict__ counts, int32_t *__restrict__ kv_index, float *__restrict__ log_pi,
    uint64_t *__restrict__ r_R, int32_t *status) {
    extern __shared__ __align__(16) uint8_t samp_smem[];
    float *s = reinterpret_cast<float *>(samp_smem);
    uint8_t *capped = samp_smem + (((size_t)nkb * 4 + 15) & ~(size_t)15);
    __shared__ uint64_t red_a[kSampleWarps];
    __shared__ int red_b[kSampleWarps];
    __shared__ int warp_cnt[kSampleWarps];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;
    const float *srow = scores + row * nkb;
    int32_t *idx_row = kv_index + row * cap;
    float *lp_row = log_pi + row * cap;

    if (n >= nkb) {  // dense budget: every block, pi = 1
        for (int j = tid; j < nkb && j < cap; j += kSampleThreads) {
            idx_row[j] = j;
            lp_row[j] = 0.f;
        }
        if (tid == 0) {
            counts[row] = min(nkb, cap);
            r_R[2 * row] = 0;
            r_R[2 * row + 1] = 0;
            if (nkb > cap) atomicOr(status, ABSA_DEVFLAG_OVERFLOW);
        }
        return;
    }

    uint64_t R = 0;
    int dummy = 0;
    for (int j = tid; j < nkb; j += kSampleThreads) {
        const float v = __ldg(srow + j);
        s[j] = v;
        capped[j] = 0;
        R += quantise_score(v);
    }
    block_sum2(R, dummy, red_a, red_b);  // also orders the shared-memory fill

    // capping fixed point: mark with (r, R), then recompute R over the rest
    int n_capped = 0;
    uint64_t r = (uint64_t)n;
    for (;;) {
        uint64_t rest = 0;
        int grew = 0;
        for (int j = tid; j < nkb; j += kSampleThreads) {
            if (capped[j]) continue;
            const uint64_t qj = quantise_score(s[j]);
            if (r * qj >= R) {
                capped[j] = 1;
                grew += 1;
            } else {
                rest += qj;
            }
        }
        block_sum2(rest, grew, red_a, red_b);
        if (grew == 0) break;
        n_capped += grew;
        r = (uint64_t)(n - n_capped);
        R = rest;
    }
    __syncthreads();

    // Poisson draws and ascending compaction, 512 blocks per round
    int base = 0;
    const uint64_t ctr0 = (uint64_t)row * (uint64_t)nkb;
    for (int j0 = 0; j0 < nkb; j0 += kSampleThreads) {
        const int j = j0 + tid;
        bool take = false;
        float lp = 0.f;
        if (j < nkb) {
            if (capped[j]) {
                take = true;
            } else {
                const uint64_t rq = r * quantise_score(s[j]);
                take = draw_taken(draw_u32(seed, ctr0 + (uint64_t)j), R, rq);
                if (take) lp = (float)log((double)rq / (double)R);
            }
        }
        const uint32_t ballot = __ballot_sync(0xffffffffu, take);
        if (lane == 0) warp_cnt[warp] = __popc(ballot);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kSampleWarps; ++w) {
            const int c = warp_cnt[w];
            before += w < warp ? c : 0;
            total += c;
        }
        if (take) {
            const int pos = base + before + __popc(ballot & ((1u << lane) - 1u));
            if (pos < cap) {
                idx_row[pos] = j;
                lp_row[pos] = lp;
            }
        }
        base += total;
        __syncthreads();
    }
    if (tid == 0) {
        counts[row] = min(base, cap);
        r_R[2 * row] = r;
        r_R[2 * row + 1] = R;
        if (base > cap) atomicOr(status, ABSA_DEVFLAG_OVERFLOW);
    }
}

cudaError_t launch_sample(const float *scores, int64_t rows, int nkb, int64_t n, uint64_t seed,
                          int cap, int32_t *counts, int32_t *kv_index, float *log_pi,
                          uint64_t *r_R, int32_t *status, cudaStream_t stream) {
    const int smem = (int)((((size_t)nkb * 4 + 15) & ~(size_t)15) + (size_t)nkb + 16);
    cudaError_t e = cudaFuncSetAttribute(absa_sample_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    absa_sample_kernel<<<(unsigned)rows, kSampleThreads, smem, stream>>>(
        scores, nkb, n, seed, cap, counts, kv_index, log_pi, r_R, status);
    return cudaGetLastError();
}

}  // namespace absa
