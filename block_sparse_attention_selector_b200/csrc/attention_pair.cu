// attention_pair.cu -- Horvitz-Thompson sparse attention for a pair of query
// blocks (2p, 2p+1) of a head over the union of their samples (K5, paired
// design), sm_100a.
//
// Method (AB-Attention summary page, "AB-Attention's three techniques", SIP
// paragraph and third paragraph): every query block attends over its own
// sampled 4-token blocks with the -ln(pi) logit shift.  Under the paired
// sampling design, query blocks 2p and 2p+1 of a head share one uniform per
// key block, so their samples nest block by block and their union is only
// 10-17% larger than each of them.  One CTA therefore gathers each key/value
// tile of the union once and runs two softmax chains on it: a block of the
// union that one of the two query blocks did not sample gets the logit bias
// -inf in that query block's chain, so each query block's output is exactly
// its own sparse attention (only the summation order differs from the
// single-block kernel).  Gathered bytes per computed FLOP fall by almost half.
// Measured on B200 this form is slower than two independent single-block
// CTAs per SM: its K/V stages wait for whole gather latencies shared by both
// chains, and every union column costs both softmax chains an exponential.
//
// Kernel design (one CTA per (b, h, query-block pair), 512 threads, one CTA
// per SM with all 512 TMEM columns):
//   setup       all threads build the union of the two plan rows in shared
//               memory: each entry's position is its index in its own row plus
//               its rank in the other row minus the shared entries before it
//               (rank by binary search, shared counts by a block scan);
//   warps 0-3   softmax of query block 2p, warps 4-7 of 2p+1 (thread = TMEM
//               lane = query row, all 64 columns of a tile), P written back
//               into the S tile's TMEM columns;
//   warps 8-10  K loaders (2-stage ring, 4-row TMA boxes) and the two bias rows
//               of each tile; warps 11-13 V loaders;
//   warp 15     MMA issuer: S_A(t) and S_B(t) from one K tile, PV_A(t) and
//               PV_B(t) from one V tile, each step issued when it is ready.
#include "absa_kernels.cuh"

namespace absa {

namespace {

constexpr int kTileKeys = kAttnTileKeys;          // key rows per tile
constexpr int kTileBlocks = kTileKeys / 4;        // 16 blocks per tile
constexpr int kKLoadWarps = 3;
constexpr int kVLoadWarps = 3;
constexpr int kLoadWarp = 8;                      // first loader warp
constexpr int kMmaWarp = 15;
constexpr int kThreads = 512;
constexpr int kStages = 2;                        // K and V ring depth
// a bias slot is rewritten once S of the tile kStages earlier is done, that is
// once the softmax of the tile kStages + 2 earlier is done
constexpr int kBiasStages = kStages <= 2 ? 4 : 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct PairSmem {
    static constexpr int kRegions = D / 64;
    static constexpr int kQRegion = 128 * 128;
    static constexpr int kKVRegion = kTileKeys * 128;
    static constexpr int kQBytes = kRegions * kQRegion;
    static constexpr int kKVBytes = kRegions * kKVRegion;
    static constexpr int kQOff = 0;                              // [A | B]
    static constexpr int kKOff = 2 * kQBytes;                    // [kStages]
    static constexpr int kVOff = kKOff + kStages * kKVBytes;     // [kStages]
    static constexpr int kBiasOff = kVOff + kStages * kKVBytes;  // [A | B][kBiasStages][64] f32
    static constexpr int kUOff = kBiasOff + 2 * kBiasStages * kTileKeys * 4;
    static constexpr int kUidOff = kUOff;                        // i32 [kPairUnionMax]
    static constexpr int kUlaOff = kUidOff + kPairUnionMax * 4;  // f32 ln pi of A (+inf: absent)
    static constexpr int kUlbOff = kUlaOff + kPairUnionMax * 4;  // f32 ln pi of B (+inf: absent)
    static constexpr int kBarOff = kUlbOff + kPairUnionMax * 4;
    static constexpr int kBytes = kBarOff + 64 * 8;
    static constexpr int kAlloc = kBytes + 1024;
    static constexpr int kStageRow = D + 8;
    // setup scratch (the two rows' ids and ln pi) lives over Q and the rings
    static_assert(4 * (kPairUnionMax / 2) * 4 <= kBiasOff, "setup scratch fits");
    static_assert(128 * kStageRow * 2 <= 2 * kStages * kKVBytes, "A staging fits the rings");
    static_assert(128 * kStageRow * 2 <= 3 * kPairUnionMax * 4, "B staging fits the union");
    static_assert(kAlloc <= 227 * 1024, "fits the shared memory of one CTA");
};

// first index in the ascending a[0..n) whose value is >= x
__device__ __forceinline__ int lower_bound_i32(const int32_t *a, int n, int32_t x) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] < x) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// O (this thread's TMEM lane, D columns from o_t) *= alpha; out of line.
template <int D>
__device__ __noinline__ void pair_rescale_o(uint32_t o_t, float alpha) {
#pragma unroll 1
    for (int ch = 0; ch < D / 16; ++ch) {
        uint32_t ov[16];
        tmem_ld16(o_t + ch * 16, ov);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
        tmem_st16(o_t + ch * 16, ov);
    }
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) absa_attention_pair_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16 *__restrict__ o, int N, int nqb,
    int nkb, float scale_log2, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ kv_index, const float *__restrict__ log_pi, int cap,
    int32_t *status) {
    using S = PairSmem<D>;
    extern __shared__ uint8_t pair_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(pair_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBarOff);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = q_full + 1;          // [kStages]
    uint64_t *k_empty = k_full + kStages;   // [kStages] S_A and S_B of the stage's tile done
    uint64_t *v_full = k_empty + kStages;   // [kStages]
    uint64_t *v_empty = v_full + kStages;   // [kStages] PV_A and PV_B of the stage's tile done
    uint64_t *s_full = v_empty + kStages;   // [2 groups][2 TMEM buffers]
    uint64_t *p_full = s_full + 4;          // [2 groups][2]
    uint64_t *pv_done = p_full + 4;         // [2 groups][2]
    uint64_t *b_full = pv_done + 4;         // [kBiasStages] both bias rows of tile j
    uint64_t *misc = b_full + kBiasStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
    int *bad_flag = reinterpret_cast<int *>(misc + 2);       // [2] per group
    int *scan = reinterpret_cast<int *>(misc + 3);           // [32] warp totals of A and B
    static_assert(1 + 4 * kStages + 12 + kBiasStages + 3 + 16 <= 64, "barrier words fit");
    int32_t *uid = reinterpret_cast<int32_t *>(sm + S::kUidOff);
    float *ula = reinterpret_cast<float *>(sm + S::kUlaOff);
    float *ulb = reinterpret_cast<float *>(sm + S::kUlbOff);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int npairs = (nqb + 1) >> 1;
    const int64_t bh = blockIdx.x / npairs;
    const int pr = blockIdx.x % npairs;
    const int qbA = 2 * pr, qbB = 2 * pr + 1;
    const bool hasB = qbB < nqb;
    const int64_t rowA = bh * nqb + qbA, rowB = rowA + 1;

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int s = 0; s < 2; ++s) {
            for (int g = 0; g < 2; ++g) {
                mbar_init(s_full + 2 * g + s, 1);
                mbar_init(p_full + 2 * g + s, 4);
                mbar_init(pv_done + 2 * g + s, 1);
            }
        }
        for (int i = 0; i < kBiasStages; ++i) mbar_init(b_full + i, kKLoadWarps);
        *abort_flag = 0;
        bad_flag[0] = 0;
        bad_flag[1] = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);

    // ---- union of the two plan rows
    int cA = __ldg(counts + rowA), cB = hasB ? __ldg(counts + rowB) : 0;
    if (cA < 0 || cA > cap) {
        if (tid == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
        cA = 0;
    }
    if (cB < 0 || cB > cap) {
        if (tid == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
        cB = 0;
    }
    int32_t *ida = reinterpret_cast<int32_t *>(sm);            // setup scratch over Q and rings
    float *lpa = reinterpret_cast<float *>(ida + cap);
    int32_t *idb = reinterpret_cast<int32_t *>(lpa + cap);
    float *lpb = reinterpret_cast<float *>(idb + cap);
    for (int i = tid; i < cA; i += kThreads) {
        ida[i] = __ldg(kv_index + rowA * cap + i);
        lpa[i] = __ldg(log_pi + rowA * cap + i);
    }
    for (int i = tid; i < cB; i += kThreads) {
        idb[i] = __ldg(kv_index + rowB * cap + i);
        lpb[i] = __ldg(log_pi + rowB * cap + i);
    }
    __syncthreads();
    // each thread takes a contiguous run of each row; pass 1 counts the run's
    // entries present in the other row, a block scan gives the runs' offsets,
    // pass 2 places the entries
    const int runA = (cA + kThreads - 1) / kThreads, runB = (cB + kThreads - 1) / kThreads;
    const int a0 = min(cA, tid * runA), a1 = min(cA, a0 + runA);
    const int b0 = min(cB, tid * runB), b1 = min(cB, b0 + runB);
    // the merge needs both rows strictly ascending (as the sampler writes
    // them); otherwise the union is the plain concatenation A then B, which
    // computes the same two attentions over more tiles
    bool run_sorted = true;
    for (int i = a0; i < a1; ++i) run_sorted &= !(i + 1 < cA && ida[i] >= ida[i + 1]);
    for (int i = b0; i < b1; ++i) run_sorted &= !(i + 1 < cB && idb[i] >= idb[i + 1]);
    const bool sorted = __syncthreads_and(run_sorted) != 0;
    int shA = 0, shB = 0;
    for (int i = a0; i < a1; ++i) {
        const int r = lower_bound_i32(idb, cB, ida[i]);
        shA += (r < cB && idb[r] == ida[i]) ? 1 : 0;
    }
    for (int i = b0; i < b1; ++i) {
        const int r = lower_bound_i32(ida, cA, idb[i]);
        shB += (r < cA && ida[r] == idb[i]) ? 1 : 0;
    }
    // exclusive block scan of (shA, shB) in thread order
    int iA = shA, iB = shB;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, iA, o2), yb = __shfl_up_sync(0xffffffffu, iB, o2);
        if (lane >= o2) {
            iA += ya;
            iB += yb;
        }
    }
    if (lane == 31) {
        scan[warp] = iA;
        scan[16 + warp] = iB;
    }
    __syncthreads();
    int baseA = 0, baseB = 0, nshared = 0;
    for (int w = 0; w < 16; ++w) {
        baseA += w < warp ? scan[w] : 0;
        baseB += w < warp ? scan[16 + w] : 0;
        nshared += scan[w];
    }
    baseA += iA - shA;
    baseB += iB - shB;
    // union size (2 * capacity <= kPairUnionMax by the host's choice)
    const int U = sorted ? cA + cB - nshared : cA + cB;
    if (!sorted) {
        for (int i = tid; i < cA; i += kThreads) {
            uid[i] = ida[i];
            ula[i] = lpa[i];
            ulb[i] = INFINITY;
        }
        for (int i = tid; i < cB; i += kThreads) {
            uid[cA + i] = idb[i];
            ula[cA + i] = INFINITY;
            ulb[cA + i] = lpb[i];
        }
    }
    for (int i = a0; i < a1 && sorted; ++i) {
        const int32_t a = ida[i];
        const int r = lower_bound_i32(idb, cB, a);
        const bool sh = r < cB && idb[r] == a;
        const int pos = i + r - baseA;
        uid[pos] = a;
        ula[pos] = lpa[i];
        ulb[pos] = sh ? lpb[r] : INFINITY;
        baseA += sh ? 1 : 0;
    }
    for (int i = b0; i < b1 && sorted; ++i) {
        const int32_t b = idb[i];
        const int r = lower_bound_i32(ida, cA, b);
        const bool sh = r < cA && ida[r] == b;
        if (!sh) {
            const int pos = i + r - baseB;
            uid[pos] = b;
            ula[pos] = INFINITY;
            ulb[pos] = lpb[i];
        }
        baseB += sh ? 1 : 0;
    }
    __syncthreads();  // the union is complete; the scratch over Q and the rings is free
    const int T = (U + kTileBlocks - 1) / kTileBlocks;
    // rows of a partial tile that no box overwrites must hold finite values;
    // the setup scratch was not bf16 data, so clear the rings unless the first
    // two tiles are full
    if (U < kStages * kTileBlocks)
        for (int i = tid; i < 2 * kStages * S::kKVBytes / 16; i += kThreads)
            reinterpret_cast<uint4 *>(sm + S::kKOff)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= kLoadWarp && warp < kLoadWarp + kKLoadWarps + kVLoadWarps) {
        // ------------------------------------------------------------ loaders
        const int lw = warp - kLoadWarp;
        const bool kside = lw < kKLoadWarps;
        const int gw = kside ? lw : lw - kKLoadWarps;
        const int gn = kside ? kKLoadWarps : kVLoadWarps;
        const int64_t row0 = bh * N;
        if (lw == 0 && lane == 0 && T > 0) {
            mbar_arrive_expect_tx(q_full, (hasB ? 2 : 1) * S::kQBytes);
            for (int g = 0; g < (hasB ? 2 : 1); ++g)
                for (int r = 0; r < S::kRegions; ++r)
                    tma_load_2d(smem_u32(sm + S::kQOff + g * S::kQBytes + r * S::kQRegion), &tm_q,
                                64 * r, (int)(row0 + (qbA + g) * 128), q_full);
        }
        constexpr int R = S::kRegions;
        const int pbox = gw + gn * lane;
        const int slot = pbox / R, reg = pbox % R;
        const bool has_box = pbox < kTileBlocks * R;
        bool ok = true;
        for (int t = 0; t < T && ok; ++t) {
            const int st = t % kStages;
            const int e = kTileBlocks * t + slot;
            int b = -1;
            float la = INFINITY, lb = INFINITY;
            if (has_box && e < U) {
                b = uid[e];
                la = ula[e];
                lb = ulb[e];
                if (b < 0 || b >= nkb) {  // an entry out of range: load block 0, zero the row(s)
                    if (la != INFINITY) atomicOr(bad_flag + 0, 1);
                    if (lb != INFINITY) atomicOr(bad_flag + 1, 1);
                    b = 0;
                }
            }
            uint64_t *empty = kside ? k_empty : v_empty;
            if (t >= kStages &&
                !__all_sync(0xffffffffu, mbar_wait(empty + st, (t / kStages - 1) & 1, status, abort_flag, 0))) {
                ok = false;
                break;
            }
            if (kside) {
                if (has_box && reg == 0) {  // the block's 4 columns in both bias rows
                    float *bias = reinterpret_cast<float *>(sm + S::kBiasOff) +
                                  (t % kBiasStages) * kTileKeys;
                    const int t0 = 4 * b;
                    float4 ba = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY), bb = ba;
                    if (b >= 0 && la != INFINITY) {
                        const float sh = -la * kLog2e;
                        ba = make_float4(t0 < N ? sh : -INFINITY, t0 + 1 < N ? sh : -INFINITY,
                                         t0 + 2 < N ? sh : -INFINITY, t0 + 3 < N ? sh : -INFINITY);
                    }
                    if (b >= 0 && lb != INFINITY) {
                        const float sh = -lb * kLog2e;
                        bb = make_float4(t0 < N ? sh : -INFINITY, t0 + 1 < N ? sh : -INFINITY,
                                         t0 + 2 < N ? sh : -INFINITY, t0 + 3 < N ? sh : -INFINITY);
                    }
                    reinterpret_cast<float4 *>(bias)[slot] = ba;
                    reinterpret_cast<float4 *>(bias + kBiasStages * kTileKeys)[slot] = bb;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(b_full + t % kBiasStages);
                    if (gw == 0)
                        mbar_arrive_expect_tx(k_full + st,
                                              min(kTileBlocks, U - kTileBlocks * t) * 512 * R);
                }
                if (b >= 0)
                    tma_load_2d(smem_u32(sm + S::kKOff + st * S::kKVBytes + reg * S::kKVRegion +
                                         slot * 512),
                                &tm_k, 64 * reg, (int)(row0 + 4 * b), k_full + st);
            } else {
                if (gw == 0 && lane == 0)
                    mbar_arrive_expect_tx(v_full + st,
                                          min(kTileBlocks, U - kTileBlocks * t) * 512 * R);
                if (b >= 0)
                    tma_load_2d(smem_u32(sm + S::kVOff + st * S::kKVBytes + reg * S::kKVRegion +
                                         slot * 512),
                                &tm_v, 64 * reg, (int)(row0 + 4 * b), v_full + st);
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        // Each query block g runs its own chain over the union tiles:
        // S_g(t) = Q_g K_t^T into TMEM buffer t % 2 of g, O_g += P_g(t) V_t.
        // The thread issues whatever step of either chain is ready (tested
        // without blocking), so the chains need not move in step:
        //   S_g(t)  once K_t has landed and PV_g(t-2) has completed (buffer free);
        //   PV_g(t) once P_g(t) is written and V_t has landed.
        // A K (V) stage is released by the commit after the second S (PV) of
        // its tile.  Giving up after about a second without progress sets the
        // timeout flag.
        if (lane == 0 && T > 0) {
            const int ng = hasB ? 2 : 1;
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTileKeys, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
            int ns[2] = {0, hasB ? 0 : T}, np[2] = {0, hasB ? 0 : T};
            bool ok = mbar_wait(q_full, 0, status, abort_flag);
            long long idle_since = clock64();
            int idle_polls = 0;
            while (ok && (np[0] < T || np[1] < T)) {
                bool progress = false;
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    if (g >= ng) break;
                    const int js = ns[g];
                    if (js < T && js < np[g] + 2 &&
                        (js < 2 || mbar_test_wait(pv_done + 2 * g + (js & 1), ((js - 2) >> 1) & 1)) &&
                        mbar_test_wait(k_full + js % kStages, (js / kStages) & 1)) {
                        tc_fence_after();
                        const int st = js % kStages;
                        const uint32_t q_s = smem_u32(sm + S::kQOff + g * S::kQBytes);
                        const uint32_t k_s = smem_u32(sm + S::kKOff + st * S::kKVBytes);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t qoff = (ks >> 2) * S::kQRegion + (ks & 3) * 32;
                            const uint32_t koff = (ks >> 2) * S::kKVRegion + (ks & 3) * 32;
                            tc_mma_f16(tmem + 256 * g + (js & 1) * kTileKeys, sw128_desc(q_s + qoff, 16, 1024),
                                       sw128_desc(k_s + koff, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                        }
                        tc_commit(s_full + 2 * g + (js & 1));
                        ns[g] = js + 1;
                        if (ns[g ^ 1] > js || ng == 1) tc_commit(k_empty + st);
                        progress = true;
                    }
                    const int j = np[g];
                    if (j < ns[g] && mbar_test_wait(p_full + 2 * g + (j & 1), (j >> 1) & 1) &&
                        mbar_test_wait(v_full + j % kStages, (j / kStages) & 1)) {
                        tc_fence_after();
                        const int st = j % kStages;
                        const uint32_t v_s = smem_u32(sm + S::kVOff + st * S::kKVBytes);
#pragma unroll
                        for (int ks = 0; ks < kTileKeys / 16; ++ks) {
                            const uint64_t bdesc = sw128_desc(v_s + (16 * ks) * 128, S::kKVRegion, 1024);
                            tc_mma_f16_tmem_a(tmem + 256 * g + 128, tmem + 256 * g + (j & 1) * kTileKeys + 8 * ks,
                                              bdesc, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
                        }
                        tc_commit(pv_done + 2 * g + (j & 1));
                        np[g] = j + 1;
                        if (np[g ^ 1] > j || ng == 1) tc_commit(v_empty + st);
                        progress = true;
                    }
                }
                if (progress) {
                    idle_since = clock64();
                    idle_polls = 0;
                } else if (++idle_polls > 16) {
                    __nanosleep(64);  // leave the issue slots to this SM partition's softmax warps
                }
                if (!progress && (clock64() - idle_since > kWaitLimitCycles || *abort_flag)) {
                    if (!*abort_flag) atomicOr(status, ABSA_DEVFLAG_TIMEOUT);
                    *abort_flag = 1;
                    ok = false;
                }
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------- softmax
        // group g = warp / 4: query block qbA + g, TMEM columns 256 g ..:
        // S/P buffers at +0 and +64, O at +128.  As in the single-block kernel:
        // x = scaled logit + bias, lazy reference max (rescale only when a
        // tile exceeds it by more than 2^8), P bf16 over the tile's own columns.
        const int g = warp >> 2;
        const int wq = warp & 3;
        const int r = wq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t tg = tmem + 256 * g;
        const uint32_t o_t = tg + 128 + lane_base;
        const float *bias_g = reinterpret_cast<const float *>(sm + S::kBiasOff) + g * kBiasStages * kTileKeys;
        const int qb = qbA + g;
        const bool active = g == 0 || hasB;
        float m_ref = -INFINITY, lsum = 0.f;
        bool ok = true;
        const int Tg = active ? T : 0;
        for (int j = 0; j < Tg; ++j) {
            const int b = j & 1;
            const uint32_t s_t = tg + lane_base + b * kTileKeys;
            ok = __all_sync(0xffffffffu, mbar_wait(s_full + 2 * g + b, (j >> 1) & 1, status, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[2][32];
            tmem_ld32(s_t, sv[0]);
            tmem_ld32(s_t + 32, sv[1]);
            tmem_wait_ld();
            const int bs = j % kBiasStages;
            ok = __all_sync(0xffffffffu, mbar_wait(b_full + bs, (j / kBiasStages) & 1, status, abort_flag));
            if (!ok) break;
            const uint32_t bias_u = smem_u32(bias_g + bs * kTileKeys);
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            const uint64_t sc2 = ((uint64_t)__float_as_uint(scale_log2) << 32) | __float_as_uint(scale_log2);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    uint64_t b01, b23;
                    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];"
                                 : "=l"(b01), "=l"(b23)
                                 : "r"(bias_u + (uint32_t)(ch * 32 + i) * 4u));
                    const uint64_t x01 = f32x2_fma(((uint64_t)sv[ch][i + 1] << 32) | sv[ch][i], sc2, b01);
                    const uint64_t x23 = f32x2_fma(((uint64_t)sv[ch][i + 3] << 32) | sv[ch][i + 2], sc2, b23);
                    sv[ch][i] = (uint32_t)x01;
                    sv[ch][i + 1] = (uint32_t)(x01 >> 32);
                    sv[ch][i + 2] = (uint32_t)x23;
                    sv[ch][i + 3] = (uint32_t)(x23 >> 32);
                    const int a = (i >> 2) & 3;
                    mx4[a] = fmaxf(mx4[a],
                                   fmaxf(fmaxf(__uint_as_float(sv[ch][i]), __uint_as_float(sv[ch][i + 1])),
                                         fmaxf(__uint_as_float(sv[ch][i + 2]), __uint_as_float(sv[ch][i + 3]))));
                }
            const float tmax = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            const bool need = tmax > m_ref + kRescaleThreshold || (m_ref == -INFINITY && tmax > -INFINITY);
            const bool any_need = j > 0 && __any_sync(0xffffffffu, need);
            const float m_new = need ? tmax : m_ref;
            const float alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - m_new);
            m_ref = m_new;
            const float moff = m_ref == -INFINITY ? 0.f : -m_ref;
            const uint64_t moff2 = ((uint64_t)__float_as_uint(moff) << 32) | __float_as_uint(moff);
            // row sum of the bf16-rounded P: the weights the PV product uses
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const uint64_t y2 = f32x2_add(((uint64_t)sv[ch][e + 1] << 32) | sv[ch][e], moff2);
                    const float p0 = ex2(__uint_as_float((uint32_t)y2));
                    const float p1 = ex2(__uint_as_float((uint32_t)(y2 >> 32)));
                    pk[e >> 1] = pack_bf16x2(p0, p1);
                    add_bf16x2_f32(pk[e >> 1], acc[2 * ((e >> 1) & 1)], acc[2 * ((e >> 1) & 1) + 1]);
                }
                tmem_st16(s_t + 16 * ch, pk);
            }
            const float tsum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            if (any_need) {  // the whole warp rescales O once PV_{j-1} is done
                ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * g + ((j - 1) & 1),
                                                       ((j - 1) >> 1) & 1, status, abort_flag));
                if (!ok) break;
                tc_fence_after();
                lsum *= alpha;
                pair_rescale_o<D>(o_t, alpha);
            }
            lsum += tsum;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 2 * g + b);
        }
        // epilogue: group A stages over the rings, group B over the union list
        constexpr int kStageRow = S::kStageRow;
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(sm + (g == 0 ? S::kKOff : S::kUOff));
        const bool bad_row = Tg > 0 && *reinterpret_cast<volatile int *>(bad_flag + g) != 0;
        const int own = g == 0 ? cA : cB;  // an empty own row is written as zeros
        if (Tg > 0 && ok && !bad_row)
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 2 * g + ((Tg - 1) & 1), ((Tg - 1) >> 1) & 1,
                                                   status, abort_flag));
        // both groups' last PVs have completed before either stages over the
        // rings or the union list (every K/V read and union read precedes them)
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const bool write = Tg > 0 && own > 0 && ok && !bad_row;
        if (write) {
            tc_fence_after();
            fence_proxy_async_smem();
            const float inv = 1.f / lsum;
#pragma unroll 1
            for (int ch = 0; ch < D / 16; ++ch) {
                uint32_t ov[16];
                tmem_ld16(o_t + ch * 16, ov);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 2; ++q8) {
                    uint4 u;
                    u.x = pack_bf16x2(__uint_as_float(ov[8 * q8]) * inv, __uint_as_float(ov[8 * q8 + 1]) * inv);
                    u.y = pack_bf16x2(__uint_as_float(ov[8 * q8 + 2]) * inv, __uint_as_float(ov[8 * q8 + 3]) * inv);
                    u.z = pack_bf16x2(__uint_as_float(ov[8 * q8 + 4]) * inv, __uint_as_float(ov[8 * q8 + 5]) * inv);
                    u.w = pack_bf16x2(__uint_as_float(ov[8 * q8 + 6]) * inv, __uint_as_float(ov[8 * q8 + 7]) * inv);
                    *reinterpret_cast<uint4 *>(stage + r * kStageRow + ch * 16 + 8 * q8) = u;
                }
            }
        }
        if (bad_row && wq == 0 && lane == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
        asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory");
        if (active) {
            const int m = min(128, N - qb * 128);
            __nv_bfloat16 *obase = o + (bh * N + (int64_t)qb * 128) * D;
            for (int c = wq * 32 + lane; c < m * (D / 8); c += 128) {
                const int rr = c / (D / 8), c8 = c % (D / 8);
                const uint4 u = write ? *reinterpret_cast<const uint4 *>(stage + rr * kStageRow + 8 * c8)
                                      : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(obase + (int64_t)rr * D + 8 * c8) = u;
            }
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

template <int D>
static cudaError_t launch_pair_d(const CUtensorMap &tq, const CUtensorMap &tk,
                                 const CUtensorMap &tv, __nv_bfloat16 *o, int64_t BH, int N,
                                 int nqb, int nkb, float scale_log2, const int32_t *counts,
                                 const int32_t *kv_index, const float *log_pi, int cap,
                                 int32_t *status, cudaStream_t stream) {
    const int smem = PairSmem<D>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(absa_attention_pair_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = BH * ((nqb + 1) / 2);
    absa_attention_pair_kernel<D><<<(unsigned)grid, kThreads, smem, stream>>>(
        tq, tk, tv, o, N, nqb, nkb, scale_log2, counts, kv_index, log_pi, cap, status);
    return cudaGetLastError();
}

cudaError_t launch_attention_pair(const CUtensorMap &tq, const CUtensorMap &tk,
                                  const CUtensorMap &tv, __nv_bfloat16 *o, int64_t BH, int N,
                                  int nqb, int nkb, int d, float softmax_scale,
                                  const int32_t *counts, const int32_t *kv_index,
                                  const float *log_pi, int cap, int32_t *status,
                                  cudaStream_t stream) {
    const float sl2 = softmax_scale * kLog2e;
    return d == 64 ? launch_pair_d<64>(tq, tk, tv, o, BH, N, nqb, nkb, sl2, counts, kv_index,
                                       log_pi, cap, status, stream)
                   : launch_pair_d<128>(tq, tk, tv, o, BH, N, nqb, nkb, sl2, counts, kv_index,
                                        log_pi, cap, status, stream);
}

}  // namespace absa
