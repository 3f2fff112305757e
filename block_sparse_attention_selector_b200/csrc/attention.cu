// attention.cu -- Horvitz-Thompson sparse attention over sampled 4-token KV
// blocks (K5) and dense attention with the same tile machinery (K6), sm_100a.
//
// Method (AB-Attention summary page, "AB-Attention's three techniques"): the
// sampled blocks enter ordinary softmax attention with the logit shift
// -ln(pi) (SIP paragraph); the 4-token blocks are gathered by index into
// full-size tensor-core tiles, tokens are not permuted (third paragraph).
//
// Kernel design (one CTA per (b, h, 128-query block), 256 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t
//   warps 4-6  loaders: cp.async gathers of 32 blocks (= 128 key rows) per
//              tile into SW128 shared-memory tiles, K and V in separate
//              2-stage rings, plus the tile's per-column logit bias
//   warp 7     TMEM owner and MMA issuer (one thread):
//              S_j = Q K_j^T  -> TMEM (two 128-column buffers)
//              O  += P_j V_j  -> TMEM (D columns), P_j bf16 in shared memory
// Softmax works in the exp2 domain: x = log2(e) * scale * (q.k) + bias with
// bias = -log2(pi) for a valid token and -inf for padding; row maxima are
// updated lazily (O is rescaled only when the max grows by more than 2^8), and
// the final O is divided by the fp32 row sum.
#include "absa_kernels.cuh"

namespace absa {

template <int D>
struct AttnSmem {
    static constexpr int kRegions = D / 64;
    static constexpr int kTile = 128 * 128;          // one SW128 region of 128 rows
    static constexpr int kQBytes = kRegions * kTile;
    static constexpr int kKVBytes = kRegions * kTile;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQBytes;              // [2] stages
    static constexpr int kVOff = kKOff + 2 * kKVBytes;         // [2] stages
    static constexpr int kPOff = kVOff + 2 * kKVBytes;         // 128 x 128 bf16
    static constexpr int kBiasOff = kPOff + 2 * kTile;         // [2][128] f32
    static constexpr int kBarOff = kBiasOff + 2 * 128 * 4;
    static constexpr int kBytes = kBarOff + 18 * 8 + 2 * 32 * 4;
    // keep one CTA per SM so that the 512-column TMEM allocation never waits
    static constexpr int kAlloc = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
};

constexpr int kLoadWarps = 3;
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kMmaWarp = 4 + kLoadWarps;
constexpr int kAttnThreads = 32 * (kMmaWarp + 1);  // 256
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D, bool DENSE>
__global__ void __launch_bounds__(kAttnThreads, 1) absa_attention_kernel(
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, __nv_bfloat16 *__restrict__ o, int N, int nqb, int nkb,
    float scale_log2, const int32_t *__restrict__ counts, const int32_t *__restrict__ kv_index,
    const float *__restrict__ log_pi, int cap, int32_t *status) {
    using S = AttnSmem<D>;
    constexpr int CH = D / 8;  // 16-byte chunks per row
    extern __shared__ uint8_t attn_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    float *bias_s = reinterpret_cast<float *>(sm + S::kBiasOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBarOff);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;   // [2]
    uint64_t *k_empty = bars + 3;  // [2]
    uint64_t *v_full = bars + 5;   // [2]
    uint64_t *v_empty = bars + 7;  // [2]
    uint64_t *s_full = bars + 9;   // [2]
    uint64_t *s_free = bars + 11;  // [2]
    uint64_t *p_full = bars + 13;
    uint64_t *p_free = bars + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 16);
    int *blk_s = reinterpret_cast<int *>(bars + 18);  // [2][32] block ids of the tile

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x / nqb;
    const int qb = blockIdx.x % nqb;
    const int64_t row = bh * nqb + qb;  // plan row
    const int m = min(128, N - qb * 128);

    if (tid == 0) {
        mbar_init(q_full, kLoadThreads);
        for (int s = 0; s < 2; ++s) {
            mbar_init(k_full + s, kLoadThreads);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, kLoadThreads);
            mbar_init(v_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(s_free + s, 4);
        }
        mbar_init(p_full, 4);
        mbar_init(p_free, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);

    // number of plan entries; reject a malformed plan row (it is written as zeros)
    int count;
    if (DENSE) {
        count = nkb;
    } else {
        count = __ldg(counts + row);
        bool bad = count < 0 || count > cap;
        if (!bad)
            for (int i = tid; i < count; i += kAttnThreads) {
                const int b = __ldg(kv_index + row * cap + i);
                bad |= (b < 0) | (b >= nkb);
            }
        if (__syncthreads_or(bad)) {
            if (tid == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
            count = 0;
        }
    }
    const int T = (count + 31) / 32;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 256;

    if (warp >= 4 && warp < 4 + kLoadWarps) {
        // ------------------------------------------------------------ loaders
        const int lt = tid - 128;
        const uint32_t q_s = smem_u32(sm + S::kQOff);
        const __nv_bfloat16 *qsrc = q + (bh * N + (int64_t)qb * 128) * D;
        for (int idx = lt; idx < 128 * CH; idx += kLoadThreads) {
            const int r = idx / CH, c = idx % CH;
            const bool ok = r < m;
            cp_async16(q_s + (c >> 3) * S::kTile + sw128_offset(r, c & 7),
                       qsrc + (int64_t)(ok ? r : 0) * D + c * 8, ok ? 16u : 0u);
        }
        cp_async_commit();
        cp_async_wait<0>();
        fence_proxy_async_smem();
        mbar_arrive(q_full);

        const __nv_bfloat16 *kh = k + bh * (int64_t)N * D;
        const __nv_bfloat16 *vh = v + bh * (int64_t)N * D;
        const int32_t *idx_row = DENSE ? nullptr : kv_index + row * cap;
        const float *lp_row = DENSE ? nullptr : log_pi + row * cap;
        bool ok = true;
        for (int j = 0; j < T && ok; ++j) {
            const int st = j & 1;
            const int nb = min(32, count - 32 * j);
            int *blk_ids = blk_s + st * 32;
            if (lt < 32) blk_ids[lt] = lt < nb ? (DENSE ? 32 * j + lt : __ldg(idx_row + 32 * j + lt)) : -1;
            asm volatile("bar.sync 2, %0;" ::"n"(kLoadThreads) : "memory");
            if (j >= 2 && !mbar_wait(k_empty + st, ((j - 2) >> 1) & 1, status, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t k_s = smem_u32(sm + S::kKOff + st * S::kKVBytes);
            for (int idx = lt; idx < 128 * CH; idx += kLoadThreads) {
                const int r = idx / CH, c = idx % CH;
                const int b = blk_ids[r >> 2];
                const int t = 4 * b + (r & 3);
                const bool valid = b >= 0 && t < N;
                cp_async16(k_s + (c >> 3) * S::kTile + sw128_offset(r, c & 7),
                           kh + (int64_t)(valid ? t : 0) * D + c * 8, valid ? 16u : 0u);
            }
            cp_async_commit();
            if (j >= 1) {  // V of the previous tile has landed: publish it
                cp_async_wait<1>();
                fence_proxy_async_smem();
                mbar_arrive(v_full + ((j - 1) & 1));
            }
            if (j >= 2 && !mbar_wait(v_empty + st, ((j - 2) >> 1) & 1, status, abort_flag)) {
                ok = false;
                break;
            }
            const uint32_t v_s = smem_u32(sm + S::kVOff + st * S::kKVBytes);
            for (int idx = lt; idx < 128 * CH; idx += kLoadThreads) {
                const int r = idx / CH, c = idx % CH;
                const int b = blk_ids[r >> 2];
                const int t = 4 * b + (r & 3);
                const bool valid = b >= 0 && t < N;
                cp_async16(v_s + (c >> 3) * S::kTile + sw128_offset(r, c & 7),
                           vh + (int64_t)(valid ? t : 0) * D + c * 8, valid ? 16u : 0u);
            }
            for (int col = lt; col < 128; col += kLoadThreads) {  // logit bias per column
                const int b = blk_ids[col >> 2];
                float bias = -INFINITY;
                if (b >= 0 && 4 * b + (col & 3) < N)
                    bias = DENSE ? 0.f : -__ldg(lp_row + 32 * j + (col >> 2)) * kLog2e;
                bias_s[st * 128 + col] = bias;
            }
            cp_async_commit();
            cp_async_wait<1>();  // K of this tile has landed
            fence_proxy_async_smem();
            mbar_arrive(k_full + st);
        }
        if (ok && T > 0) {
            cp_async_wait<0>();
            fence_proxy_async_smem();
            mbar_arrive(v_full + ((T - 1) & 1));
        }
        cp_async_wait<0>();
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
            const uint32_t q_s = smem_u32(sm + S::kQOff);
            const uint32_t p_s = smem_u32(sm + S::kPOff);
            bool ok = T == 0 || mbar_wait(q_full, 0, status, abort_flag);
            auto issue_pv = [&](int jj) -> bool {
                const int st = jj & 1;
                if (!mbar_wait(v_full + st, (jj >> 1) & 1, status, abort_flag)) return false;
                if (!mbar_wait(p_full, jj & 1, status, abort_flag)) return false;
                tc_fence_after();
                const uint32_t v_s = smem_u32(sm + S::kVOff + st * S::kKVBytes);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t a = sw128_desc(p_s + (ks >> 2) * S::kTile + (ks & 3) * 32, 16, 1024);
                    const uint64_t b = sw128_desc(v_s + ks * 2048, S::kTile, 1024);
                    tc_mma_f16(tmem_o, a, b, idesc_o, (jj > 0 || ks > 0) ? 1u : 0u);
                }
                tc_commit(p_free);
                tc_commit(v_empty + st);
                return true;
            };
            for (int j = 0; ok && j < T; ++j) {
                const int st = j & 1, b = j & 1;
                if (!mbar_wait(k_full + st, (j >> 1) & 1, status, abort_flag)) break;
                if (j >= 2 && !mbar_wait(s_free + b, ((j - 2) >> 1) & 1, status, abort_flag)) break;
                tc_fence_after();
                const uint32_t k_s = smem_u32(sm + S::kKOff + st * S::kKVBytes);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * S::kTile + (ks & 3) * 32;
                    tc_mma_f16(tmem + b * 128, sw128_desc(q_s + off, 16, 1024),
                               sw128_desc(k_s + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                }
                tc_commit(s_full + b);
                tc_commit(k_empty + st);
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok && T > 0) issue_pv(T - 1);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int r = tid;  // query row = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t p_s = smem_u32(sm + S::kPOff);
        float m_ref = -INFINITY, lsum = 0.f;
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            ok = __all_sync(0xffffffffu, mbar_wait(s_full + b, (j >> 1) & 1, status, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) tmem_ld32(tmem + lane_base + b * 128 + ch * 32, sv[ch]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_free + b);
            ok = __all_sync(0xffffffffu, mbar_wait(v_full + b, (j >> 1) & 1, status, abort_flag));
            if (!ok) break;
            const float *bias = bias_s + b * 128;
            float tmax = -INFINITY;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch)
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    const float4 bb = *reinterpret_cast<const float4 *>(bias + ch * 32 + i);
                    const float x0 = __fmaf_rn(__uint_as_float(sv[ch][i]), scale_log2, bb.x);
                    const float x1 = __fmaf_rn(__uint_as_float(sv[ch][i + 1]), scale_log2, bb.y);
                    const float x2 = __fmaf_rn(__uint_as_float(sv[ch][i + 2]), scale_log2, bb.z);
                    const float x3 = __fmaf_rn(__uint_as_float(sv[ch][i + 3]), scale_log2, bb.w);
                    sv[ch][i] = __float_as_uint(x0);
                    sv[ch][i + 1] = __float_as_uint(x1);
                    sv[ch][i + 2] = __float_as_uint(x2);
                    sv[ch][i + 3] = __float_as_uint(x3);
                    tmax = fmaxf(tmax, fmaxf(fmaxf(x0, x1), fmaxf(x2, x3)));
                }
            if (j == 0) m_ref = tmax;
            const bool need = j > 0 && tmax > m_ref + kRescaleThreshold;
            const bool any_need = __any_sync(0xffffffffu, need);
            const float m_new = need ? tmax : m_ref;
            const float alpha = ex2(m_ref - m_new);
            m_ref = m_new;
            if (j >= 1) {  // PV of the previous tile is done: P buffer free, O stable
                ok = __all_sync(0xffffffffu, mbar_wait(p_free, (j - 1) & 1, status, abort_flag));
                if (!ok) break;
            }
            const float moff = -m_ref;
            float acc = 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
                for (int g = 0; g < 4; ++g) {  // 8 columns = one 16-byte chunk
                    float p[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        p[e] = ex2(__uint_as_float(sv[ch][g * 8 + e]) + moff);
                        acc += p[e];
                    }
                    const int col = ch * 32 + g * 8;
                    const uint32_t dst = p_s + (col >> 6) * S::kTile + sw128_offset(r, (col >> 3) & 7);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                                 "r"(pack_bf16x2(p[0], p[1])), "r"(pack_bf16x2(p[2], p[3])),
                                 "r"(pack_bf16x2(p[4], p[5])), "r"(pack_bf16x2(p[6], p[7]))
                                 : "memory");
                }
            }
            if (any_need) {  // lazy rescale of the running output by exp2(m_old - m_new)
                tc_fence_after();
                lsum *= alpha;
#pragma unroll
                for (int ch = 0; ch < D / 32; ++ch) {
                    uint32_t ov[32];
                    tmem_ld32(tmem_o + lane_base + ch * 32, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                    tmem_st32(tmem_o + lane_base + ch * 32, ov);
                }
                tmem_wait_st();
            }
            lsum += acc;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // epilogue: O / lsum -> bf16, valid rows only
        __nv_bfloat16 *orow = o + (bh * N + (int64_t)qb * 128 + r) * D;
        if (T > 0 && ok) {
            ok = __all_sync(0xffffffffu, mbar_wait(p_free, (T - 1) & 1, status, abort_flag));
        }
        if (T > 0 && ok) {
            tc_fence_after();
            const float inv = 1.f / lsum;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ov[32];
                tmem_ld32(tmem_o + lane_base + ch * 32, ov);
                tmem_wait_ld();
                if (r < m) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint4 u;
                        u.x = pack_bf16x2(__uint_as_float(ov[8 * g + 0]) * inv,
                                          __uint_as_float(ov[8 * g + 1]) * inv);
                        u.y = pack_bf16x2(__uint_as_float(ov[8 * g + 2]) * inv,
                                          __uint_as_float(ov[8 * g + 3]) * inv);
                        u.z = pack_bf16x2(__uint_as_float(ov[8 * g + 4]) * inv,
                                          __uint_as_float(ov[8 * g + 5]) * inv);
                        u.w = pack_bf16x2(__uint_as_float(ov[8 * g + 6]) * inv,
                                          __uint_as_float(ov[8 * g + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + ch * 32 + 8 * g) = u;
                    }
                }
            }
        } else if (T == 0 && r < m) {
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < CH; ++c) *reinterpret_cast<uint4 *>(orow + c * 8) = z;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int D, bool DENSE>
static cudaError_t launch_attention_d(const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                                      const __nv_bfloat16 *v, __nv_bfloat16 *o, int64_t BH, int N,
                                      int nqb, int nkb, float scale_log2, const int32_t *counts,
                                      const int32_t *kv_index, const float *log_pi, int cap,
                                      int32_t *status, cudaStream_t stream) {
    const int smem = AttnSmem<D>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(absa_attention_kernel<D, DENSE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    absa_attention_kernel<D, DENSE><<<(unsigned)(BH * nqb), kAttnThreads, smem, stream>>>(
        q, k, v, o, N, nqb, nkb, scale_log2, counts, kv_index, log_pi, cap, status);
    return cudaGetLastError();
}

cudaError_t launch_attention(bool dense, const __nv_bfloat16 *q, const __nv_bfloat16 *k,
                             const __nv_bfloat16 *v, __nv_bfloat16 *o, int64_t BH, int N, int nqb,
                             int nkb, int d, float softmax_scale, const int32_t *counts,
                             const int32_t *kv_index, const float *log_pi, int cap,
                             int32_t *status, cudaStream_t stream) {
    const float sl2 = softmax_scale * kLog2e;
    if (d == 64)
        return dense ? launch_attention_d<64, true>(q, k, v, o, BH, N, nqb, nkb, sl2, counts,
                                                    kv_index, log_pi, cap, status, stream)
                     : launch_attention_d<64, false>(q, k, v, o, BH, N, nqb, nkb, sl2, counts,
                                                     kv_index, log_pi, cap, status, stream);
    return dense ? launch_attention_d<128, true>(q, k, v, o, BH, N, nqb, nkb, sl2, counts,
                                                 kv_index, log_pi, cap, status, stream)
                 : launch_attention_d<128, false>(q, k, v, o, BH, N, nqb, nkb, sl2, counts,
                                                  kv_index, log_pi, cap, status, stream);
}

}  // namespace absa
