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
// One CTA of d threads per (head, group): thread e owns dimension e, so the
// loads of a token row are coalesced; two passes over the group (the second
// from L1/L2) give the variance without cancellation.  Every K and V byte is
// read once from HBM: 4 N d bytes per head.
#include "absa_kernels.cuh"

namespace absa {

template <int D>
__global__ void __launch_bounds__(D) absa_group_stats_kernel(
    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v, int N, int ngroups,
    __nv_bfloat16 *__restrict__ mu, __nv_bfloat16 *__restrict__ nu, float *__restrict__ gvar,
    int32_t *__restrict__ gcnt) {
    __shared__ float red[D / 32];
    const int e = threadIdx.x;
    const int64_t bh = blockIdx.x / ngroups;
    const int g = blockIdx.x % ngroups;
    const int t0 = 4 * kRemGroupBlocks * g;
    const int t1 = min(N, t0 + 4 * kRemGroupBlocks);
    const int n = t1 - t0;
    const __nv_bfloat16 *kh = k + (bh * N + t0) * D + e;
    const __nv_bfloat16 *vh = v + (bh * N + t0) * D + e;
    float sk = 0.f, sv = 0.f;
#pragma unroll 4
    for (int t = 0; t < n; ++t) {
        sk += __bfloat162float(kh[(int64_t)t * D]);
        sv += __bfloat162float(vh[(int64_t)t * D]);
    }
    const float inv = 1.f / (float)n;
    const float m = sk * inv;
    float ss = 0.f;
#pragma unroll 4
    for (int t = 0; t < n; ++t) {
        const float dk = __bfloat162float(kh[(int64_t)t * D]) - m;
        ss = fmaf(dk, dk, ss);
    }
    const int64_t out = bh * ngroups + g;
    mu[out * D + e] = __float2bfloat16_rn(m);
    nu[out * D + e] = __float2bfloat16_rn(sv * inv);
    float var = ss * inv;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) var += __shfl_xor_sync(0xffffffffu, var, o);
    if ((e & 31) == 0) red[e >> 5] = var;
    __syncthreads();
    if (e == 0) {
        float tv = 0.f;
#pragma unroll
        for (int w = 0; w < D / 32; ++w) tv += red[w];
        gvar[out] = tv / (float)D;
        gcnt[out] = n;
    }
}

cudaError_t launch_group_stats(const __nv_bfloat16 *k, const __nv_bfloat16 *v, int64_t BH, int N,
                               int d, int ngroups, __nv_bfloat16 *mu, __nv_bfloat16 *nu,
                               float *gvar, int32_t *gcnt, cudaStream_t stream) {
    const int64_t grid = BH * ngroups;
    if (d == 64)
        absa_group_stats_kernel<64><<<(unsigned)grid, 64, 0, stream>>>(k, v, N, ngroups, mu, nu,
                                                                      gvar, gcnt);
    else
        absa_group_stats_kernel<128><<<(unsigned)grid, 128, 0, stream>>>(k, v, N, ngroups, mu, nu,
                                                                        gvar, gcnt);
    return cudaGetLastError();
}

}  // namespace absa
