// attention.cu -- Horvitz-Thompson sparse attention over sampled 4-token KV
// blocks (K5) and dense attention with the same tile machinery (K6), sm_100a.
//
// Method (AB-Attention summary page, "AB-Attention's three techniques"): the
// sampled blocks enter ordinary softmax attention with the logit shift
// -ln(pi) (SIP paragraph); the 4-token blocks are gathered by index into
// full-size tensor-core tiles, tokens are not permuted (third paragraph).
//
// Kernel design (one CTA per (b, h, 128-query block), 320 threads, about 98 KB
// of shared memory and 256 TMEM columns, so that two CTAs -- two independent
// softmax -> P -> PV chains -- share each SM and fill each other's gaps):
//   warps 0-3   softmax, one warpgroup (thread = TMEM lane = query row) over
//               all 64 columns of every S tile; it writes P (bf16) back into
//               the tile's own TMEM columns
//   warps 4-8   loaders: TMA gathers of 16 blocks (= 64 key rows) per tile into
//               SW128 shared-memory tiles; warps 4-6 fill the 2-stage K ring
//               and the tile's per-column logit bias (4-slot ring), warps 7-8
//               the 2-stage V ring, each group at its own pace
//   warp 9      TMEM owner and MMA issuer (one thread):
//               S_j = Q K_j^T  -> TMEM buffer j % 2 (64 columns)
//               O  += P_j V_j  (A = P_j read from TMEM, B = V_j in shared
//               memory) -> one D-column accumulator
// Softmax works in the exp2 domain: x = log2(e) * scale * (q.k) + bias with
// bias = -log2(pi) for a valid token and -inf for padding; the row maximum is
// updated lazily (O is rescaled only when the max grows by more than 2^8), and
// the final O is divided by the fp32 sum of the bf16-rounded P, the weights
// the PV product used (a row dominated by a few tokens then returns their
// values without the rounding of P showing).
//
// Remainder mode (ESTRA page, summary and figure: the selected pairs exact,
// the rest from group averages with a variance-calibrated correction): the
// plan's tiles run with a zero bias, then tiles of 64 group representatives
// (mean keys and values of 32-block groups, loaded as 64-row boxes) follow in
// the same softmax chain, each with the bias log2 of its tokens outside the
// plan row and the term |q|^2 * s^2 var / 2 added to its logits.
#include "absa_kernels.cuh"

namespace absa {

constexpr int kTileKeys = kAttnTileKeys;               // key rows per tile
constexpr int kTileBlocks = kTileKeys / 4;             // 4-token blocks per tile
constexpr int kSoftmaxWarps = 4;                       // one warpgroup
constexpr int kKLoadWarps = 3;                         // K ring and bias
constexpr int kVLoadWarps = 2;                         // V ring
constexpr int kLoadWarp = kSoftmaxWarps;               // first loader warp
constexpr int kLoadWarps = kKLoadWarps + kVLoadWarps;
constexpr int kMmaWarp = kLoadWarp + kLoadWarps;       // 9
constexpr int kAttnThreads = 32 * (kMmaWarp + 1);      // 320
constexpr int kBiasStages = 4;
constexpr int kLoaderPolls = 0;                        // loaders sleep at once when they wait
constexpr int kTmemCols = 256;                         // S/P [2][64], O at column 128
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct AttnSmem {
    static constexpr int kRegions = D / 64;              // 64-element SW128 regions
    static constexpr int kQRegion = 128 * 128;           // 128 rows of 128 bytes
    static constexpr int kKVRegion = kTileKeys * 128;    // 64 rows of 128 bytes
    static constexpr int kQBytes = kRegions * kQRegion;
    static constexpr int kKVBytes = kRegions * kKVRegion;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQBytes;               // [2] stages
    static constexpr int kVOff = kKOff + 2 * kKVBytes;          // [2] stages
    static constexpr int kBiasOff = kVOff + 2 * kKVBytes;       // [4][64] f32
    static constexpr int kBarOff = kBiasOff + kBiasStages * kTileKeys * 4;
    static constexpr int kBytes = kBarOff + 32 * 8;
    static constexpr int kAlloc = kBytes + 1024;  // room to align the tiles to 1024 bytes
    // the output tile is staged over the (by then idle) K and V rings: rows of
    // D bf16 with a 16-byte pad against bank conflicts
    static constexpr int kStageRow = D + 8;
    static_assert(128 * kStageRow * 2 <= 4 * kKVBytes, "output staging fits the rings");
};

// O (this thread's TMEM lane, D columns from o_t) *= alpha.  Kept out of line:
// it runs only when a row maximum grows by more than 2^8, and inlined its
// registers would add to the softmax loop's.
template <int D>
__device__ __noinline__ void rescale_o(uint32_t o_t, float alpha) {
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

// Loaders.  Sparse mode: a tile's 16 blocks x (d/64) column regions are 4-row
// TMA boxes (512 bytes each) placed at rows 4i..4i+3 of the SW128 tile; the
// box swizzle follows the shared-memory address, so a box in the upper half
// of a 1024-byte atom lands in that half's chunk order.  A group's boxes are
// spread over its warps (box p goes to warp p % n): a single warp sustains
// only a fraction of the gather rate of several.  Block ids and log(pi) of
// the next tile are prefetched while the current tile is issued.  Dense
// mode: one 64-row box per region from one lane.
// The logit bias of tile t is written together with K_t into slot t % 4 of
// its own ring (every K loader warp arrives on b_full after writing its
// columns), so the softmax of a tile never waits for that tile's V.
template <int D, bool DENSE, bool REM>
__global__ void __launch_bounds__(kAttnThreads, 2) absa_attention_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16 *__restrict__ k,
    const __nv_bfloat16 *__restrict__ v, __nv_bfloat16 *__restrict__ o, int N, int nqb,
    int nkb, float scale_log2, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ kv_index, const float *__restrict__ log_pi, int cap,
    int32_t *status, const __grid_constant__ RemainderArgs rem) {
    using S = AttnSmem<D>;
    extern __shared__ uint8_t attn_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
    float *bias_s = reinterpret_cast<float *>(sm + S::kBiasOff);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + S::kBarOff);
    uint64_t *q_full = bars + 0;
    uint64_t *k_full = bars + 1;    // [2]
    uint64_t *k_empty = bars + 3;   // [2]
    uint64_t *v_full = bars + 5;    // [2]
    uint64_t *v_empty = bars + 7;   // [2]
    uint64_t *s_full = bars + 9;    // [2] S_j in TMEM buffer j % 2
    uint64_t *p_full = bars + 11;   // [2] P_j written over S_j
    uint64_t *pv_done = bars + 13;  // [2] PV_j complete: buffer j % 2 free, O stable
    uint64_t *b_full = bars + 15;   // [4] logit bias of tile j in slot j % 4
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 19);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 20);
    int *bad_flag = reinterpret_cast<int *>(bars + 21);  // a plan entry out of range
    // remainder mode: per tile slot the representatives' variance terms
    // (64 floats after the bias ring) and the plan's tokens per group
    float *cvar_s = reinterpret_cast<float *>(sm + S::kBytes);
    int *gsel = reinterpret_cast<int *>(sm + S::kBytes + kBiasStages * kTileKeys * 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x / nqb;
    const int qb = blockIdx.x % nqb;
    const int64_t row = bh * nqb + qb;  // plan row
    const int m = min(128, N - qb * 128);

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(p_full + s, kSoftmaxWarps);
            mbar_init(pv_done + s, 1);
        }
        for (int i = 0; i < kBiasStages; ++i) mbar_init(b_full + i, DENSE ? 1 : kKLoadWarps);
        static_assert(!(DENSE && REM), "the remainder mode extends the sparse mode");
        *abort_flag = 0;
        *bad_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, kTmemCols);

    // Number of plan entries: a count outside [0, cap] rejects the row (it is
    // written as zeros).  Entries outside [0, NKB) are caught by the loaders,
    // which read them anyway: such an entry loads block 0 instead and the row
    // is written as zeros at the end.
    int count;
    bool count_bad = false;
    if (DENSE) {
        count = nkb;
    } else {
        count = __ldg(counts + row);
        if (count < 0 || count > cap) {
            if (tid == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
            count = 0;
            count_bad = true;
        }
    }
    const int Ts = (count + kTileBlocks - 1) / kTileBlocks;  // tiles of plan blocks
    // remainder mode: then one tile per 64 group representatives (none for a
    // rejected row, which is written as zeros)
    const int T = Ts + (REM && !count_bad ? (rem.ngroups + kTileKeys - 1) / kTileKeys : 0);
    if (REM) {  // tokens of the plan's blocks per group
        for (int g = tid; g < rem.ngroups; g += kAttnThreads) gsel[g] = 0;
        __syncthreads();
        const int32_t *ir = kv_index + row * cap;
        for (int e0 = tid; e0 < count; e0 += 4 * kAttnThreads) {  // 4 entry loads in flight
            int bq[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                bq[u] = e0 + u * kAttnThreads < count ? __ldg(ir + e0 + u * kAttnThreads) : -1;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (bq[u] >= 0 && bq[u] < nkb)
                    atomicAdd(&gsel[bq[u] / kRemGroupBlocks], min(4, N - 4 * bq[u]));
        }
    }
    // Rows of a partial tile that no box overwrites must hold finite values
    // (P = 0 there, and 0 * NaN would poison O).  After its first use a ring
    // stage holds finite stale rows, so only a row whose first two tiles are
    // not both full needs the rings cleared (dense tiles past N are zero-filled
    // by the TMA unit).
    if (!DENSE && count < 2 * kTileBlocks)
        for (int i = tid; i < 4 * S::kKVBytes / 16; i += kAttnThreads)
            reinterpret_cast<uint4 *>(sm + S::kKOff)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_o = tmem + 128;

    if (warp >= kLoadWarp && warp < kLoadWarp + kLoadWarps) {
        // ------------------------------------------------------------ loaders
        const int lw = warp - kLoadWarp;      // 0..5
        const bool kside = lw < kKLoadWarps;  // K group (K tiles and bias) or V group
        const int gw = kside ? lw : lw - kKLoadWarps;         // warp within the group
        const int gn = kside ? kKLoadWarps : kVLoadWarps;      // warps in the group
        const int64_t row0 = bh * N;          // first token row of this head
        if (lw == 0 && lane == 0 && T > 0) {
            mbar_arrive_expect_tx(q_full, S::kQBytes);
            const uint32_t q_s = smem_u32(sm + S::kQOff);
            for (int r = 0; r < S::kRegions; ++r)
                tma_load_2d(q_s + r * S::kQRegion, &tm_q, 64 * r, (int)(row0 + qb * 128), q_full);
        }
        const int32_t *idx_row = DENSE ? nullptr : kv_index + row * cap;
        const float *lp_row = DENSE ? nullptr : log_pi + row * cap;
        // box p = gw + gn * lane of a tile: block slot p / R, region p % R
        constexpr int R = S::kRegions;
        const int pbox = gw + gn * lane;
        const int slot = pbox / R, reg = pbox % R;
        const bool has_box = pbox < kTileBlocks * R;
        // this lane's plan entry (block id, log pi) in tile t; -1 past the end
        auto entry = [&](int t, int &b, float &lp) {
            b = -1;
            lp = 0.f;
            const int e = kTileBlocks * t + slot;
            if (!DENSE && has_box && e < count) {
                b = __ldg(idx_row + e);
                lp = __ldg(lp_row + e);
            }
        };
        // An entry of tile t present in the plan but outside [0, NKB) loads
        // block 0 instead and marks the row (checked where the entry is used,
        // a tile after its load, so the check adds no load latency).
        auto checked = [&](int t, int b) -> int {
            if (!DENSE && has_box && kTileBlocks * t + slot < count && (b < 0 || b >= nkb)) {
                atomicOr(bad_flag, 1);
                return 0;
            }
            return b;
        };
        // K_t and the logit bias of tile t (bias slot t % 4; a slot is
        // rewritten only after S_{t-2} has completed, which the MMA issues
        // only once PV_{t-4}, and so the softmax of tile t-4, is done)
        auto issue_k = [&](int t, int b, float lpv) -> bool {
            const int st = t & 1;
            b = checked(t, b);
            if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(k_empty + st, ((t - 2) >> 1) & 1,
                                                             status, abort_flag, kLoaderPolls)))
                return false;
            float *bias = bias_s + (t % kBiasStages) * kTileKeys;
            const uint32_t k_s = smem_u32(sm + S::kKOff + st * S::kKVBytes);
            if (REM && t >= Ts) {
                // a tile of 64 group representatives: mean keys, log2 of the
                // tokens left outside the plan, and the variance term
                const int g0 = kTileKeys * (t - Ts);
                const int64_t gb = bh * rem.ngroups;
                if (lw == 0) {
                    float bb[2], cc[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int g = g0 + 2 * lane + h;
                        const bool in = g < rem.ngroups;
                        const int left = in ? __ldg(rem.gcnt + gb + g) - gsel[g] : 0;
                        bb[h] = left > 0 ? log2f((float)left) : -INFINITY;
                        cc[h] = in ? rem.var_coef * __ldg(rem.gvar + gb + g) : 0.f;
                    }
                    reinterpret_cast<float2 *>(bias)[lane] = make_float2(bb[0], bb[1]);
                    reinterpret_cast<float2 *>(cvar_s + (t % kBiasStages) * kTileKeys)[lane] =
                        make_float2(cc[0], cc[1]);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(b_full + t % kBiasStages);
                    if (lw == 0) {
                        mbar_arrive_expect_tx(k_full + st, S::kKVBytes);
                        for (int r = 0; r < R; ++r)
                            tma_load_2d(k_s + r * S::kKVRegion, &rem.tm_mu, 64 * r,
                                        (int)(gb + g0), k_full + st);
                    }
                }
            } else if (DENSE) {
                if (lw == 0) {
                    float2 bb;
                    const int t0 = kTileKeys * t + 2 * lane;
                    bb.x = t0 < N ? 0.f : -INFINITY;
                    bb.y = t0 + 1 < N ? 0.f : -INFINITY;
                    reinterpret_cast<float2 *>(bias)[lane] = bb;
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(b_full + t % kBiasStages);
                        mbar_arrive_expect_tx(k_full + st, S::kKVBytes);
                        for (int r = 0; r < R; ++r)
                            tma_load_2d(k_s + r * S::kKVRegion, &tm_k, 64 * r,
                                        (int)(row0 + kTileKeys * t), k_full + st);
                    }
                }
            } else {
                if (has_box && reg == 0) {  // logit bias of the block's 4 columns
                    float4 bb = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
                    if (b >= 0) {
                        const float sh = REM ? 0.f : -lpv * kLog2e;  // remainder mode: no HT shift
                        const int t0 = 4 * b;
                        bb.x = t0 < N ? sh : -INFINITY;
                        bb.y = t0 + 1 < N ? sh : -INFINITY;
                        bb.z = t0 + 2 < N ? sh : -INFINITY;
                        bb.w = t0 + 3 < N ? sh : -INFINITY;
                    }
                    reinterpret_cast<float4 *>(bias)[slot] = bb;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(b_full + t % kBiasStages);
                    if (gw == 0)
                        mbar_arrive_expect_tx(k_full + st,
                                              min(kTileBlocks, count - kTileBlocks * t) * 512 * R);
                }
                if (b >= 0)
                    tma_load_2d(k_s + reg * S::kKVRegion + slot * 512, &tm_k, 64 * reg,
                                (int)(row0 + 4 * b), k_full + st);
            }
            return true;
        };
        auto issue_v = [&](int t, int b) -> bool {
            const int st = t & 1;
            b = checked(t, b);
            if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait(v_empty + st, ((t - 2) >> 1) & 1,
                                                             status, abort_flag, kLoaderPolls)))
                return false;
            const uint32_t v_s = smem_u32(sm + S::kVOff + st * S::kKVBytes);
            if (REM && t >= Ts) {  // the representatives' mean values
                if (gw == 0 && lane == 0) {
                    mbar_arrive_expect_tx(v_full + st, S::kKVBytes);
                    for (int r = 0; r < R; ++r)
                        tma_load_2d(v_s + r * S::kKVRegion, &rem.tm_nu, 64 * r,
                                    (int)(bh * rem.ngroups + kTileKeys * (t - Ts)), v_full + st);
                }
            } else if (DENSE) {
                if (gw == 0 && lane == 0) {
                    mbar_arrive_expect_tx(v_full + st, S::kKVBytes);
                    for (int r = 0; r < R; ++r)
                        tma_load_2d(v_s + r * S::kKVRegion, &tm_v, 64 * r,
                                    (int)(row0 + kTileKeys * t), v_full + st);
                }
            } else {
                if (gw == 0 && lane == 0)
                    mbar_arrive_expect_tx(v_full + st,
                                          min(kTileBlocks, count - kTileBlocks * t) * 512 * R);
                if (b >= 0)
                    tma_load_2d(v_s + reg * S::kKVRegion + slot * 512, &tm_v, 64 * reg,
                                (int)(row0 + 4 * b), v_full + st);
            }
            return true;
        };
        // Each group walks the tiles at its own pace (the K group also writes
        // the bias); plan entries are fetched one tile ahead.
        int b0, b1;
        float l0, l1;
        entry(0, b0, l0);
        bool ok = true;
        for (int t = 0; t < T && ok; ++t) {
            entry(t + 1, b1, l1);
            ok = kside ? issue_k(t, b0, l0) : issue_v(t, b0);
            b0 = b1;
            l0 = l1;
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer
        // One thread issues, in a fixed order, S_0, S_1 and then for every
        // tile j: O += P_j V_j, and (once PV_j has completed, so that P_j in
        // TMEM buffer j % 2 has been read) S_{j+2} = Q K_{j+2}^T into that
        // buffer.  Each step waits (bounded) for its operands.
        if (lane == 0 && T > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTileKeys, 0);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 1);
            const uint32_t q_s = smem_u32(sm + S::kQOff);
            auto issue_s = [&](int js) -> bool {
                const int st = js & 1;
                if (!mbar_wait(k_full + st, (js >> 1) & 1, status, abort_flag)) return false;
                tc_fence_after();
                const uint32_t k_s = smem_u32(sm + S::kKOff + st * S::kKVBytes);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t qoff = (ks >> 2) * S::kQRegion + (ks & 3) * 32;
                    const uint32_t koff = (ks >> 2) * S::kKVRegion + (ks & 3) * 32;
                    tc_mma_f16(tmem + st * kTileKeys, sw128_desc(q_s + qoff, 16, 1024),
                               sw128_desc(k_s + koff, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                }
                tc_commit(s_full + st);
                tc_commit(k_empty + st);
                return true;
            };
            auto issue_pv = [&](int j) -> bool {
                const int st = j & 1;
                if (!mbar_wait(p_full + st, (j >> 1) & 1, status, abort_flag)) return false;
                if (!mbar_wait(v_full + st, (j >> 1) & 1, status, abort_flag)) return false;
                tc_fence_after();
                const uint32_t v_s = smem_u32(sm + S::kVOff + st * S::kKVBytes);
#pragma unroll
                for (int ks = 0; ks < kTileKeys / 16; ++ks) {  // 16 keys = 8 P columns per step
                    const uint64_t bdesc =
                        sw128_desc(v_s + (16 * ks) * 128, S::kKVRegion, 1024);
                    tc_mma_f16_tmem_a(tmem_o, tmem + st * kTileKeys + 8 * ks, bdesc, idesc_o,
                                      (j > 0 || ks > 0) ? 1u : 0u);
                }
                tc_commit(pv_done + st);
                tc_commit(v_empty + st);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, status, abort_flag) && issue_s(0);
            if (ok && T > 1) ok = issue_s(1);
            for (int j = 0; j < T; ++j) {
                ok = issue_pv(j);
                if (ok && j + 2 < T)
                    ok = mbar_wait(pv_done + (j & 1), (j >> 1) & 1, status, abort_flag) &&
                         issue_s(j + 2);
            }
        }
    } else {
        // ------------------------------------------------------------- softmax
        // Thread = TMEM lane = query row; one online softmax over the 64
        // columns of every S tile.  P_j (bf16) goes into the first 32 columns
        // of S_j's own TMEM buffer (two keys per column), where the PV MMA
        // reads it.
        const int r = warp * 32 + lane;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t o_t = tmem_o + lane_base;
        float m_ref = -INFINITY, lsum = 0.f;
        bool ok = true;
        // remainder mode: |q_r|^2 for the representatives' variance term, from
        // this row of the Q tile (the swizzle only permutes the row's 16-byte
        // chunks; lane r starts at chunk r so that the lanes spread over banks)
        float *qn_s = reinterpret_cast<float *>(gsel + kRemMaxGroups);  // [128] |q_r|^2
        if (REM && T > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, status, abort_flag));
            float qn = 0.f;
#pragma unroll 1
            for (int rr = 0; rr < S::kRegions; ++rr)
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(
                        sm + S::kQOff + rr * S::kQRegion + r * 128 + ((c + r) & 7) * 16);
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
                        qn = fmaf(lo, lo, fmaf(hi, hi, qn));
                    }
                }
            // read back per group tile, divided by the logit scale (no term at scale 0)
            qn_s[r] = scale_log2 != 0.f ? qn / scale_log2 : 0.f;
        }
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            const uint32_t s_t = tmem + lane_base + b * kTileKeys;
            ok = __all_sync(0xffffffffu, mbar_wait(s_full + b, (j >> 1) & 1, status, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t sv[2][32];
            tmem_ld32(s_t, sv[0]);
            tmem_ld32(s_t + 32, sv[1]);
            tmem_wait_ld();
            const int bs = j % kBiasStages;
            ok = __all_sync(0xffffffffu,
                            mbar_wait(b_full + bs, (j / kBiasStages) & 1, status, abort_flag));
            if (!ok) break;
            const uint32_t bias_u = smem_u32(bias_s + bs * kTileKeys);
            const uint32_t cvar_u = REM ? smem_u32(cvar_s + bs * kTileKeys) : 0u;
            if (REM && j >= Ts) {
                // representatives: fold |q_r|^2 c_g into S (S += |q_r|^2 c_g / scale),
                // so that the loop below stays the one of the plan's tiles
                const float qs = qn_s[r];
                const uint64_t qs2 = ((uint64_t)__float_as_uint(qs) << 32) | __float_as_uint(qs);
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        uint64_t c01, c23;
                        asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];"
                                     : "=l"(c01), "=l"(c23)
                                     : "r"(cvar_u + (uint32_t)(ch * 32 + i) * 4u));
                        const uint64_t s01 = f32x2_fma(c01, qs2, ((uint64_t)sv[ch][i + 1] << 32) | sv[ch][i]);
                        const uint64_t s23 = f32x2_fma(c23, qs2, ((uint64_t)sv[ch][i + 3] << 32) | sv[ch][i + 2]);
                        sv[ch][i] = (uint32_t)s01;
                        sv[ch][i + 1] = (uint32_t)(s01 >> 32);
                        sv[ch][i + 2] = (uint32_t)s23;
                        sv[ch][i + 3] = (uint32_t)(s23 >> 32);
                    }
            }
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            const uint64_t sc2 =
                ((uint64_t)__float_as_uint(scale_log2) << 32) | __float_as_uint(scale_log2);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                for (int i = 0; i < 32; i += 4) {
                    uint64_t b01, b23;
                    asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];"
                                 : "=l"(b01), "=l"(b23)
                                 : "r"(bias_u + (uint32_t)(ch * 32 + i) * 4u));
                    const uint64_t x01 =
                        f32x2_fma(((uint64_t)sv[ch][i + 1] << 32) | sv[ch][i], sc2, b01);
                    const uint64_t x23 =
                        f32x2_fma(((uint64_t)sv[ch][i + 3] << 32) | sv[ch][i + 2], sc2, b23);
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
            // lazy max: keep the reference unless the tile exceeds it by 2^8;
            // a row whose columns so far were all padding has m_ref = -inf
            const bool need =
                tmax > m_ref + kRescaleThreshold || (m_ref == -INFINITY && tmax > -INFINITY);
            const bool any_need = j > 0 && __any_sync(0xffffffffu, need);
            const float m_new = need ? tmax : m_ref;
            const float alpha = m_ref == -INFINITY ? 0.f : ex2(m_ref - m_new);
            m_ref = m_new;
            const float moff = m_ref == -INFINITY ? 0.f : -m_ref;
            const uint64_t moff2 = ((uint64_t)__float_as_uint(moff) << 32) | __float_as_uint(moff);
            // row sum of the bf16-rounded P: the weights the PV product uses
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {  // P_j in two halves of 16 columns (32 keys)
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const uint64_t y2 =
                        f32x2_add(((uint64_t)sv[ch][e + 1] << 32) | sv[ch][e], moff2);
                    const float p0 = ex2(__uint_as_float((uint32_t)y2));
                    const float p1 = ex2(__uint_as_float((uint32_t)(y2 >> 32)));
                    pk[e >> 1] = pack_bf16x2(p0, p1);
                    add_bf16x2_f32(pk[e >> 1], acc[2 * ((e >> 1) & 1)], acc[2 * ((e >> 1) & 1) + 1]);
                }
                tmem_st16(s_t + 16 * ch, pk);
            }
            const float tsum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            if (any_need) {  // lazy rescale of O by exp2(m_old - m_new) once PV_{j-1} is done
                ok = __all_sync(0xffffffffu, mbar_wait(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1,
                                                       status, abort_flag));
                if (!ok) break;
                tc_fence_after();
                lsum *= alpha;
                rescale_o<D>(o_t, alpha);
            }
            lsum += tsum;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + b);
        }
        // epilogue: o = O / l.  Every softmax thread reaches the barriers below
        // exactly once.
        constexpr int kStageRow = S::kStageRow;
        __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(sm + S::kKOff);
        // a plan entry out of range (seen by the loaders before their last
        // arrival on b_full, which every softmax warp has waited for)
        const bool bad_row = !DENSE && T > 0 && *reinterpret_cast<volatile int *>(bad_flag) != 0;
        if (T > 0 && ok && !bad_row)
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done + ((T - 1) & 1), ((T - 1) >> 1) & 1,
                                                   status, abort_flag));
        const bool write = T > 0 && ok && !bad_row;
        if (write) {
            // the last PV has completed, and with it every MMA that read the
            // rings; every TMA copy into them has been waited for
            tc_fence_after();
            fence_proxy_async_smem();  // generic writes after the rings' async-proxy use
            const float inv = 1.f / lsum;
#pragma unroll 1
            for (int ch = 0; ch < D / 16; ++ch) {
                uint32_t ov[16];
                tmem_ld16(o_t + ch * 16, ov);
                tmem_wait_ld();
#pragma unroll
                for (int g = 0; g < 2; ++g) {
                    uint4 u;
                    u.x = pack_bf16x2(__uint_as_float(ov[8 * g]) * inv, __uint_as_float(ov[8 * g + 1]) * inv);
                    u.y = pack_bf16x2(__uint_as_float(ov[8 * g + 2]) * inv, __uint_as_float(ov[8 * g + 3]) * inv);
                    u.z = pack_bf16x2(__uint_as_float(ov[8 * g + 4]) * inv, __uint_as_float(ov[8 * g + 5]) * inv);
                    u.w = pack_bf16x2(__uint_as_float(ov[8 * g + 6]) * inv, __uint_as_float(ov[8 * g + 7]) * inv);
                    *reinterpret_cast<uint4 *>(stage + r * kStageRow + ch * 16 + 8 * g) = u;
                }
            }
        }
        if (bad_row && tid == 0) atomicOr(status, ABSA_DEVFLAG_BAD_PLAN);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kSoftmaxWarps) : "memory");
        // coalesced rows: consecutive threads write consecutive 16-byte chunks
        __nv_bfloat16 *obase = o + (bh * N + (int64_t)qb * 128) * D;
        for (int c = tid; c < m * (D / 8); c += 32 * kSoftmaxWarps) {
            const int rr = c / (D / 8), c8 = c % (D / 8);
            const uint4 u = write ? *reinterpret_cast<const uint4 *>(stage + rr * kStageRow + 8 * c8)
                                  : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(obase + (int64_t)rr * D + 8 * c8) = u;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D, bool DENSE, bool REM>
static cudaError_t launch_attention_d(const CUtensorMap &tq, const CUtensorMap &tk,
                                      const CUtensorMap &tv, const __nv_bfloat16 *k,
                                      const __nv_bfloat16 *v, __nv_bfloat16 *o, int64_t BH, int N,
                                      int nqb, int nkb, float scale_log2, const int32_t *counts,
                                      const int32_t *kv_index, const float *log_pi, int cap,
                                      int32_t *status, const RemainderArgs &rem,
                                      cudaStream_t stream) {
    // remainder mode: the variance-term ring and the per-group plan tokens follow
    const int smem =
        AttnSmem<D>::kAlloc + (REM ? kBiasStages * kTileKeys * 4 + kRemMaxGroups * 4 + 128 * 4 : 0);
    cudaError_t e = cudaFuncSetAttribute(absa_attention_kernel<D, DENSE, REM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // two CTAs per SM: ask for the largest shared-memory carveout
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(absa_attention_kernel<D, DENSE, REM>,
                                 cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    absa_attention_kernel<D, DENSE, REM><<<(unsigned)(BH * nqb), kAttnThreads, smem, stream>>>(
        tq, tk, tv, k, v, o, N, nqb, nkb, scale_log2, counts, kv_index, log_pi, cap, status, rem);
    return cudaGetLastError();
}

cudaError_t launch_attention(bool dense, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, const __nv_bfloat16 *k,
                             const __nv_bfloat16 *v, __nv_bfloat16 *o, int64_t BH, int N, int nqb,
                             int nkb, int d, float softmax_scale, const int32_t *counts,
                             const int32_t *kv_index, const float *log_pi, int cap,
                             int32_t *status, cudaStream_t stream, const RemainderArgs *rem) {
    const float sl2 = softmax_scale * kLog2e;
    RemainderArgs none;
    memset(&none, 0, sizeof(none));
    const RemainderArgs &ra = rem ? *rem : none;
#define ABSA_LAUNCH(DD, DN, RM)                                                                    \
    return launch_attention_d<DD, DN, RM>(tq, tk, tv, k, v, o, BH, N, nqb, nkb, sl2, counts,      \
                                          kv_index, log_pi, cap, status, ra, stream)
    if (d == 64) {
        if (dense) ABSA_LAUNCH(64, true, false);
        if (rem) ABSA_LAUNCH(64, false, true);
        ABSA_LAUNCH(64, false, false);
    }
    if (dense) ABSA_LAUNCH(128, true, false);
    if (rem) ABSA_LAUNCH(128, false, true);
    ABSA_LAUNCH(128, false, false);
#undef ABSA_LAUNCH
}

}  // namespace absa
