// select.cu -- IBCS block selector on sm_100a (AB-Attention summary page,
// "AB-Attention's three techniques", IBCS paragraph):
//   K1 (in K2)             mean key of every 4-token block, split hi+lo fp16
//   K2 absa_kmeans_kernel  per-128-query-block Lloyd k-means in shared memory,
//                          plus the key-block means of the same token range
// (the block score from these centroids is in score.cu)
#include "absa_kernels.cuh"

namespace absa {

// ------------------------------------------------------------------------ K1

// Mean of nt (1..4) token rows of one 8-element chunk (tokens summed in
// ascending order in fp32, then times 1/4 or divided by nt) stored as
// mean = hi + lo with hi = fp16(mean), lo = fp16(mean - hi) (round to nearest
// even, clamped to +-65504; hi + lo is within about 2^-22 of the mean).  The
// k-means kernel runs this for the 32 key blocks of its own 128-token range.
__device__ __forceinline__ void pool_chunk(const uint4 (&u)[4], int nt, uint4 &hi_u, uint4 &lo_u) {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        if (t < nt) {
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u[t]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                acc[2 * e] += f.x;
                acc[2 * e + 1] += f.y;
            }
        }
    }
    uint32_t *hp = reinterpret_cast<uint32_t *>(&hi_u);
    uint32_t *lp = reinterpret_cast<uint32_t *>(&lo_u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float m0 = nt == 4 ? acc[2 * e] * 0.25f : __fdiv_rn(acc[2 * e], (float)nt);
        const float m1 = nt == 4 ? acc[2 * e + 1] * 0.25f : __fdiv_rn(acc[2 * e + 1], (float)nt);
        const __half h0 = f16_sat(m0), h1 = f16_sat(m1);
        const __half l0 = f16_sat(m0 - __half2float(h0));
        const __half l1 = f16_sat(m1 - __half2float(h1));
        hp[e] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
        lp[e] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
    }
}

// ------------------------------------------------------------------------ K2

// One CTA (128 threads) per query block.  fp32 arithmetic in a fixed order:
//  load:                  every thread issues all of its 16-byte loads of the
//                         block before storing any of them (one memory
//                         latency per block), into rows of pitch D+8 bf16
//                         (an odd number of 16-byte units, so 8 threads
//                         reading 16 bytes of 8 different rows hit 8
//                         different bank groups);
//  assignment (thread i): dist_c = sum over ascending e of fma(x-mu, x-mu, .),
//                         two clusters per packed f32x2 instruction (each lane
//                         rounds exactly like the scalar operation), argmin
//                         with ties to the lowest c; row i is read 8 dims at
//                         a time;
//  update:                members of each cluster ranked in ascending i with
//                         warp ballots; the clusters are split in contiguous
//                         runs of about equal membership over 256/D groups of
//                         D/2 threads, thread dl of a group summing dims 2dl
//                         and 2dl+1 (one bf16 pair of each member row) over
//                         ascending i, with the next 8 members' loads in
//                         flight while the current 8 are added;
//                         mu = sum / count (IEEE division); an empty cluster
//                         keeps mu.
template <int D>
struct KmeansSmem {
    static constexpr int kRow = D + 8;                  // bf16 row pitch: an odd number of 16 B units
    static constexpr int kX = 0;                        // bf16 [128][D+8]
    static constexpr int kMu = kX + 128 * kRow * 2;     // f32 [D][8] (transposed)
    static constexpr int kList = kMu + D * 8 * 4;       // i32 [8][128] member lists
    static constexpr int kCnt = kList + 8 * 128 * 4;    // i32 [4 warps][8] + [8] totals
    static constexpr int kBytes = kCnt + (4 * 8 + 8) * 4;
    static_assert(((kRow * 2 / 16) & 1) == 1 && (kRow * 2) % 16 == 0, "row pitch");
    static_assert(kMu % 16 == 0 && kList % 16 == 0, "alignment");
};

template <int D>
__global__ void __launch_bounds__(128, 5) absa_kmeans_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k, int N, int nqb,
    int nkb, int iters, float *__restrict__ mu_out, __half *__restrict__ mu_hi,
    __half *__restrict__ mu_lo, float *__restrict__ w_out, uint8_t *__restrict__ assign_out,
    __half *__restrict__ kbar_hi, __half *__restrict__ kbar_lo) {
    using S = KmeansSmem<D>;
    constexpr int NC = 8;
    extern __shared__ __align__(16) uint8_t kms[];
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(kms + S::kX);
    float *mut = reinterpret_cast<float *>(kms + S::kMu);
    int *mlist = reinterpret_cast<int *>(kms + S::kList);
    int *wcnt = reinterpret_cast<int *>(kms + S::kCnt);  // [warp][c]
    int *cnt_s = wcnt + 4 * NC;                          // [c]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;  // (b*H + h)*nqb + qb
    const int64_t bh = row / nqb;
    const int qb = (int)(row % nqb);
    const int m = min(128, N - qb * 128);
    const __nv_bfloat16 *src = q + (bh * N + (int64_t)qb * 128) * D;

    constexpr int XR = S::kRow;      // bf16 per row
    constexpr int XW = XR / 2;       // 32-bit words per row
    constexpr int CPR = D / 8;       // 16-byte units per row of q
    {
        const uint4 *src4 = reinterpret_cast<const uint4 *>(src);
        uint4 v[CPR];
#pragma unroll
        for (int u = 0; u < CPR; ++u) {  // 128 * CPR units, CPR per thread
            const int idx = tid + 128 * u;
            if (idx / CPR < m) v[u] = __ldg(src4 + idx);
        }
#pragma unroll
        for (int u = 0; u < CPR; ++u) {
            const int idx = tid + 128 * u, r = idx / CPR, c = idx % CPR;
            if (r < m) *reinterpret_cast<uint4 *>(xs + r * XR + c * 8) = v[u];
        }
    }
    {
        // K1: pooled keys of the same 128-token range, key blocks 32 qb .. 32 qb + 31,
        // one chunk per thread at a time with its four loads issued first (two at a
        // time spill at the 96 registers of five CTAs per SM)
        constexpr int UPT = CPR / 4;  // 32 blocks x CPR chunks over 128 threads
        constexpr int BATCH = 1;
        const int jb0 = qb * 32;
        const int nblk = min(32, nkb - jb0);
        const __nv_bfloat16 *ksrc = k + (bh * N + (int64_t)qb * 128) * D;
#pragma unroll
        for (int i0 = 0; i0 < UPT; i0 += BATCH) {
            uint4 kv[BATCH][4];
            int nt[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int u = tid + 128 * (i0 + i), blk = u / CPR, c = u % CPR;
                nt[i] = blk < nblk ? min(4, N - 4 * (jb0 + blk)) : 0;
#pragma unroll
                for (int t = 0; t < 4; ++t)
                    if (t < nt[i])
                        kv[i][t] = __ldg(reinterpret_cast<const uint4 *>(ksrc + (int64_t)(4 * blk + t) * D) + c);
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                if (nt[i] == 0) continue;
                const int u = tid + 128 * (i0 + i), blk = u / CPR, c = u % CPR;
                uint4 hi_u, lo_u;
                pool_chunk(kv[i], nt[i], hi_u, lo_u);
                const int64_t o = (bh * nkb + jb0 + blk) * (int64_t)D + c * 8;
                *reinterpret_cast<uint4 *>(kbar_hi + o) = hi_u;
                *reinterpret_cast<uint4 *>(kbar_lo + o) = lo_u;
            }
        }
    }
    __syncthreads();
    for (int idx = tid; idx < NC * D; idx += 128) {
        const int c = idx / D, e = idx % D;
        mut[e * NC + c] = __bfloat162float(xs[((c * m) / NC) * XR + e]);
    }
    __syncthreads();

    const uint32_t *xs32 = reinterpret_cast<const uint32_t *>(xs);
    for (int it = 0; it < iters; ++it) {
        int a = 0;
        if (tid < m) {
            uint64_t dist[NC / 2] = {0, 0, 0, 0};  // (+0.f, +0.f) pairs
            const __nv_bfloat16 *xrow = xs + tid * XR;
#pragma unroll 2
            for (int c8 = 0; c8 < CPR; ++c8) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xrow + c8 * 8);
                const uint32_t wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const int e = c8 * 8 + h;
                    const uint32_t pair = wv[h >> 1];
                    const uint32_t xb = (h & 1) ? (pair & 0xFFFF0000u) : (pair << 16);
                    const uint64_t x2 = (uint64_t)xb | ((uint64_t)xb << 32);
                    const ulonglong2 m01 = *reinterpret_cast<const ulonglong2 *>(mut + e * NC);
                    const ulonglong2 m45 = *reinterpret_cast<const ulonglong2 *>(mut + e * NC + 4);
                    const uint64_t mc[NC / 2] = {m01.x, m01.y, m45.x, m45.y};
#pragma unroll
                    for (int c = 0; c < NC / 2; ++c) {
                        const uint64_t diff = f32x2_sub(x2, mc[c]);
                        dist[c] = f32x2_fma(diff, diff, dist[c]);
                    }
                }
            }
            float bd = __uint_as_float((uint32_t)dist[0]);
#pragma unroll
            for (int c = 1; c < NC; ++c) {
                const float dc = __uint_as_float((uint32_t)(dist[c >> 1] >> (32 * (c & 1))));
                if (dc < bd) {
                    bd = dc;
                    a = c;
                }
            }
        }
        // rank of query tid among the members of its cluster (ascending i)
        const bool valid = tid < m;
        uint32_t my_ballot = 0;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const uint32_t bal = __ballot_sync(0xffffffffu, valid && a == c);
            if (lane == 0) wcnt[warp * NC + c] = __popc(bal);
            if (a == c) my_ballot = bal;
        }
        __syncthreads();
        if (valid) {
            int pos = __popc(my_ballot & ((1u << lane) - 1u));
            for (int w = 0; w < warp; ++w) pos += wcnt[w * NC + a];
            mlist[a * 128 + pos] = tid;
        }
        if (tid < NC) cnt_s[tid] = wcnt[tid] + wcnt[NC + tid] + wcnt[2 * NC + tid] + wcnt[3 * NC + tid];
        __syncthreads();
        {
            constexpr int G = 256 / D;  // groups of D/2 threads (whole warps)
            const int g = tid / (D / 2), dl = tid % (D / 2);
            const uint32_t *xw = xs32 + dl;  // word dl of row 0
            int before = 0;
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                const int n = cnt_s[c];
                const int owner = min(G - 1, ((2 * before + n) * G) / (2 * m));
                before += n;
                if (n == 0 || owner != g) continue;
                const int *ml = mlist + c * 128;
                float acc0 = 0.f, acc1 = 0.f;
                auto add8 = [&](const uint32_t (&pv)[8]) {
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        acc0 = __fadd_rn(acc0, __uint_as_float(pv[u] << 16));
                        acc1 = __fadd_rn(acc1, __uint_as_float(pv[u] & 0xFFFF0000u));
                    }
                };
                auto load8 = [&](int t0, uint32_t (&pv)[8]) {
                    const int4 ia = *reinterpret_cast<const int4 *>(ml + t0);
                    const int4 ib = *reinterpret_cast<const int4 *>(ml + t0 + 4);
                    const int id[8] = {ia.x, ia.y, ia.z, ia.w, ib.x, ib.y, ib.z, ib.w};
#pragma unroll
                    for (int u = 0; u < 8; ++u) pv[u] = xw[id[u] * XW];
                };
                int t = 0;
                if (n >= 8) {
                    uint32_t cur[8];
                    load8(0, cur);
                    for (t = 8; t + 8 <= n; t += 8) {
                        uint32_t nxt[8];
                        load8(t, nxt);
                        add8(cur);
#pragma unroll
                        for (int u = 0; u < 8; ++u) cur[u] = nxt[u];
                    }
                    add8(cur);
                }
                for (; t < n; ++t) {
                    const uint32_t pv = xw[ml[t] * XW];
                    acc0 = __fadd_rn(acc0, __uint_as_float(pv << 16));
                    acc1 = __fadd_rn(acc1, __uint_as_float(pv & 0xFFFF0000u));
                }
                mut[(2 * dl) * NC + c] = __fdiv_rn(acc0, (float)n);
                mut[(2 * dl + 1) * NC + c] = __fdiv_rn(acc1, (float)n);
            }
        }
        __syncthreads();
    }
    if (tid < NC) w_out[row * NC + tid] = __fdiv_rn((float)cnt_s[tid], (float)m);
    for (int idx = tid; idx < NC * D; idx += 128) {
        const int c = idx / D, e = idx % D;
        const float v = mut[e * NC + c];
        const int64_t o = (row * NC + c) * D + e;
        mu_out[o] = v;
        const __half h = f16_sat(v);
        mu_hi[o] = h;
        mu_lo[o] = f16_sat(v - __half2float(h));
    }
    // final assignment: member lists of the last round
    for (int c = 0; c < NC; ++c)
        for (int t = tid; t < cnt_s[c]; t += 128) assign_out[row * 128 + mlist[c * 128 + t]] = (uint8_t)c;
    if (tid >= m) assign_out[row * 128 + tid] = (uint8_t)255;
}

// ------------------------------------------------------------------ launchers

template <int D>
static cudaError_t launch_kmeans_d(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int64_t BH,
                                   int N, int nqb, int nkb, int iters, float *mu, __half *mu_hi,
                                   __half *mu_lo, float *w, uint8_t *assign, __half *kbar_hi,
                                   __half *kbar_lo, cudaStream_t stream) {
    const int smem = KmeansSmem<D>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(absa_kmeans_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    absa_kmeans_kernel<D><<<(unsigned)(BH * nqb), 128, smem, stream>>>(
        q, k, N, nqb, nkb, iters, mu, mu_hi, mu_lo, w, assign, kbar_hi, kbar_lo);
    return cudaGetLastError();
}

cudaError_t launch_kmeans_pool(const __nv_bfloat16 *q, const __nv_bfloat16 *k, int64_t BH, int N,
                               int nqb, int nkb, int d, int iters, float *mu, __half *mu_hi,
                               __half *mu_lo, float *w, uint8_t *assign, __half *kbar_hi,
                               __half *kbar_lo, cudaStream_t stream) {
    return d == 64 ? launch_kmeans_d<64>(q, k, BH, N, nqb, nkb, iters, mu, mu_hi, mu_lo, w, assign,
                                         kbar_hi, kbar_lo, stream)
                   : launch_kmeans_d<128>(q, k, BH, N, nqb, nkb, iters, mu, mu_hi, mu_lo, w,
                                          assign, kbar_hi, kbar_lo, stream);
}

}  // namespace absa
