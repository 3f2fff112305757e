// remainder.cu -- group statistics for the ESTRA-style remainder of the
// sparse attention (K7a), sm_100a.
//
// Method (ESTRA page, summary and figure: keys grouped, the rest of the
// attention approximated from group averages with a variance-calibrated
// correction of the representatives' weights).  For every head and every
// group g of kRemGroupBlocks consecutive 4-token key blocks (128 tokens):
//   mu_g  = mean key over the group's tokens        (bf16, an MMA operand)
//   nu_g  = mean value                              (bf16, an MMA operand)
//   var_g = (1/d) sum_e mean_t (k_te - mu_ge)^2     (f32)
//   n_g   = tokens in the group (the last group of a head can be short).
// The attention kernel's remainder mode weighs each representative by the
// tokens of its group outside the plan and adds s^2 |q|^2 var_g / 2 to its
// logit (the moment identity E exp(X) = exp(E X + Var X / 2) of a Gaussian
// X = s q.k, with the key spread taken as isotropic).
//
// One CTA of 256 threads per (head, group): thread (r, c) owns the 8
// dimensions of 16-byte chunk c of token rows r, r + R, ... (R = 256 / (d/8)
// rows at a time), so every load is a coalesced 16-byte vector; the column
// sums meet in shared memory, and a second pass over the group (from L1/L2)
// gives the variance without cancellation.  Every K and V byte is read once
// from HBM: 4 N d bytes per head.
#include "absa_kernels.cuh"

namespace absa {

constexpr int kStatsThreads = 256;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        f[2 * h] = __uint_as_float(w[h] << 16);
        f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(kStatsThreads) absa_group_stats_kernel(
    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v, int N, int ngroups,
    __nv_bfloat16 *__restrict__ mu, __nv_bfloat16 *__restrict__ nu, float *__restrict__ gvar,
    int32_t *__restrict__ gcnt) {
    constexpr int C = D / 8;                 // 16-byte chunks per token row
    constexpr int R = kStatsThreads / C;     // token rows per step
    __shared__ float col_k[R][D], col_v[R][D];
    __shared__ float mean_k[D];
    __shared__ float red[kStatsThreads / 32];
    const int tid = threadIdx.x, r = tid / C, c = tid % C;
    const int64_t bh = blockIdx.x / ngroups;
    const int g = blockIdx.x % ngroups;
    const int t0 = 4 * kRemGroupBlocks * g;
    const int n = min(N, t0 + 4 * kRemGroupBlocks) - t0;
    const uint4 *k4 = reinterpret_cast<const uint4 *>(k + (bh * N + t0) * D) + c;
    const uint4 *v4 = reinterpret_cast<const uint4 *>(v + (bh * N + t0) * D) + c;
    float sk[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, sv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int t = r; t < n; t += R) {
        float fk[8], fv[8];
        bf16x8_to_f32(__ldg(k4 + (int64_t)t * C), fk);
        bf16x8_to_f32(__ldg(v4 + (int64_t)t * C), fv);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            sk[i] += fk[i];
            sv[i] += fv[i];
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        col_k[r][8 * c + i] = sk[i];
        col_v[r][8 * c + i] = sv[i];
    }
    __syncthreads();
    const float inv = 1.f / (float)n;
    const int64_t out = bh * ngroups + g;
    if (tid < D) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int j = 0; j < R; ++j) {
            a += col_k[j][tid];
            b += col_v[j][tid];
        }
        mean_k[tid] = a * inv;
        mu[out * D + tid] = __float2bfloat16_rn(a * inv);
        nu[out * D + tid] = __float2bfloat16_rn(b * inv);
    }
    __syncthreads();
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = mean_k[8 * c + i];
    float ss = 0.f;
#pragma unroll 4
    for (int t = r; t < n; t += R) {
        float fk[8];
        bf16x8_to_f32(__ldg(k4 + (int64_t)t * C), fk);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float dk = fk[i] - m[i];
            ss = fmaf(dk, dk, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
        float tv = 0.f;
#pragma unroll
        for (int w = 0; w < kStatsThreads / 32; ++w) tv += red[w];
        gvar[out] = tv * inv / (float)D;
        gcnt[out] = n;
    }
}

cudaError_t launch_group_stats(const __nv_bfloat16 *k, const __nv_bfloat16 *v, int64_t BH, int N,
                               int d, int ngroups, __nv_bfloat16 *mu, __nv_bfloat16 *nu,
                               float *gvar, int32_t *gcnt, cudaStream_t stream) {
    const int64_t grid = BH * ngroups;
    if (d == 64)
        absa_group_stats_kernel<64><<<(unsigned)grid, kStatsThreads, 0, stream>>>(
            k, v, N, ngroups, mu, nu, gvar, gcnt);
    else
        absa_group_stats_kernel<128><<<(unsigned)grid, kStatsThreads, 0, stream>>>(
            k, v, N, ngroups, mu, nu, gvar, gcnt);
    return cudaGetLastError();
}

}  // namespace absa
