// sample.cu -- SIP sampler on sm_100a (AB-Attention summary page, "AB-Attention's
// three techniques", SIP paragraph): inclusion probability proportional to the
// block score, the top blocks capped at pi = 1, the rest keeping a nonzero
// chance, sum pi = budget; draws from a counter-based hash, either
// independent per block (Poisson design) or one per row for systematic
// sampling (exactly `budget` blocks; the paragraph fixes the probabilities,
// not the design); ascending compaction of the taken blocks with their ln(pi).
//
// Integer formulation (exact, so every ordering of the reductions gives the
// same plan): q_j = max(1, floor(s_j 2^32)); capping fixed point on
// (r, R) = (n - |C|, sum_{j not in C} q_j) with u64 block reductions; draw
// u_j * R < (r q_j) 2^32 compared exactly.  u_j is output ctr+1 of the
// SplitMix64 generator started from state mix(seed), ctr = row * NKB + j;
// the paired design draws query blocks 2p and 2p+1 of a head from the
// counters of block 2p, so their samples nest block by block.
#include "absa_kernels.cuh"

namespace absa {

// q - 1 as a u32 (q = max(1, floor(s 2^32)) <= 2^32).
__device__ __forceinline__ uint32_t quantise_m1(float s) {
    const float x = s * 4294967296.0f;  // exact power-of-two scaling
    if (!(x >= 1.0f)) return 0u;        // NaN, negative, or below one unit
    if (x >= 4294967296.0f) return 0xFFFFFFFFu;
    return __float2uint_rz(x) - 1u;     // floor for 1 <= x < 2^32
}

// Threshold t - 1 of "q >= t" on q - 1 as a u32, or `never` when t - 1 exceeds
// every q - 1 (q <= 2^32).
__device__ __forceinline__ uint32_t q_threshold_m1(uint64_t t, bool &never) {
    never = t - 1 > 0xFFFFFFFFull;
    return never ? 0xFFFFFFFFu : (uint32_t)(t - 1);
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;  // SplitMix64 increment

// Upper 32 bits of the SplitMix64 output function of z.  Only the high word
// of the second product and of the last xor-shift is formed: with
// z = hi 2^32 + lo, the high word of z * c mod 2^64 is
// hi32(lo * c_lo) + lo * c_hi + hi * c_lo (mod 2^32), and the high word of
// z ^ (z >> 31) is hi ^ (hi >> 31).
__device__ __forceinline__ uint32_t splitmix64_hi32(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    const uint32_t lo = (uint32_t)z, hi = (uint32_t)(z >> 32);
    const uint32_t h = __umulhi(lo, 0x133111EBu) + lo * 0x94D049BBu + hi * 0x133111EBu;
    return h ^ (h >> 31);
}

// Candidate list for the capping rounds after the first (see the kernel).
constexpr int kCandMax = 2048;

// u * R < rq * 2^32 exactly (u < 2^32, R < 2^48, rq < 2^48): with
// R = Rh 2^32 + Rl, u R = (u Rh + hi32(u Rl)) 2^32 + lo32(u Rl), so the
// comparison reduces to u Rh + hi32(u Rl) < rq.
__device__ __forceinline__ bool draw_taken(uint32_t u, uint32_t Rh, uint32_t Rl, uint64_t rq) {
    return (uint64_t)u * Rh + __umulhi(u, Rl) < rq;
}

// (x + y) mod R and (x - y) mod R for x, y < R < 2^49.
__device__ __forceinline__ uint64_t addmod(uint64_t x, uint64_t y, uint64_t R) {
    const uint64_t z = x + y;
    return z >= R ? z - R : z;
}
__device__ __forceinline__ uint64_t submod(uint64_t x, uint64_t y, uint64_t R) {
    return x >= y ? x - y : x + R - y;
}

// Block-wide sum of a u64 and an int over WARPS warps; result broadcast to every thread.
template <int WARPS>
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
    for (int w = 0; w < WARPS; ++w) {
        a += red_a[w];
        b += red_b[w];
    }
}

// One CTA per plan row (b,h,qb); the grid covers rows row0 .. row0+gridDim-1
// of the whole problem (scores and plan pointers start at row0, the hash
// counter uses the global row).  Key blocks are handled in groups of 32 (one
// per lane); warp w owns a contiguous run of groups, so the taken blocks of
// warp w all precede those of warp w+1 and one scan of the 8 warp counts
// places every entry.  Shared memory: q_j - 1 as u32 per block, one capped
// word and one taken word (ballots) per group, and the candidate list.
//
// Capping: the first round (r = n, R = sum q) runs over every block and also
// lists the blocks with 2 n q_j >= R_total, i.e. q_j at least half of the
// first threshold R/r.  The threshold only decreases from round to round, and
// while it stays at or above that half every block a later round caps is on
// the list, so warp 0 runs those rounds over the list alone.  If the list
// overflows or the threshold falls below the half, the remaining rounds scan
// every block.  Either way the rounds are exactly those of the definition.
template <int WARPS>
__global__ void __launch_bounds__(32 * WARPS, WARPS == 8 ? 5 : WARPS == 16 ? 2 : 1) absa_sample_kernel(
    const float *__restrict__ scores, int nkb, int64_t n, uint64_t seed, int cap,
    int32_t *__restrict__ counts, int32_t *__restrict__ kv_index, float *__restrict__ log_pi,
    uint64_t *__restrict__ r_R, int32_t *status, int64_t row0, int design, int nqb) {
    constexpr int kSampleWarps = WARPS;
    constexpr int kSampleThreads = 32 * WARPS;
    extern __shared__ __align__(16) uint32_t samp_smem[];
    const int ngroups = (nkb + 31) >> 5;
    const int ngp = (ngroups + 7) & ~7;             // groups rounded up to whole 256-block
                                                    // super-groups (systematic pass)
    uint32_t *qm1 = samp_smem;                      // [ngp*32]
    uint32_t *capw = samp_smem + ngp * 32;          // [ngp]
    uint32_t *takew = capw + ngp;                   // [ngp]
    uint32_t *cand = takew + ngp;                   // [kCandMax]
    __shared__ uint64_t red_a[kSampleWarps];
    __shared__ int red_b[kSampleWarps];
    __shared__ int warp_cnt[kSampleWarps];
    __shared__ int n_cand;
    __shared__ uint64_t fin_R;
    __shared__ int fin_capped, fin_full;

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

    const int per_warp = (ngroups + kSampleWarps - 1) / kSampleWarps;
    const int g0 = warp * per_warp;
    const int g1 = min(ngroups, g0 + per_warp);

    // quantise once; R = sum of all q_j
    if (tid == 0) n_cand = 0;
    uint64_t R = 0;
    int dummy = 0;
    for (int g = g0; g < g1; g += 8) {  // 8 loads in flight per lane
        float sv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = (g + u) * 32 + lane;
            sv[u] = (g + u < g1 && j < nkb) ? __ldg(srow + j) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = (g + u) * 32 + lane;
            if (g + u < g1 && j < nkb) {
                const uint32_t qm = quantise_m1(sv[u]);
                qm1[j] = qm;
                R += (uint64_t)qm + 1;
            }
        }
    }
    block_sum2<WARPS>(R, dummy, red_a, red_b);
    const uint64_t R0 = R;
    const uint64_t nn = (uint64_t)n;

    // round 1 over every block (r = n), listing the candidates for later rounds:
    // n q >= R0 <=> q >= ceil(R0 / n), and 2 n q >= R0 <=> q >= ceil(R0 / (2 n)),
    // compared on q - 1 in 32 bits
    const uint32_t below = (1u << lane) - 1u;
    bool never_cap, never_cand;
    const uint32_t t_cap = q_threshold_m1((R0 + nn - 1) / nn, never_cap);
    const uint32_t t_cand = q_threshold_m1((R0 + 2 * nn - 1) / (2 * nn), never_cand);
    uint64_t capsum = 0;
    int capcnt = 0;
    for (int g = g0; g < g1; ++g) {
        const int j = g * 32 + lane;
        bool newcap = false, is_cand = false;
        if (j < nkb) {
            const uint32_t qm = qm1[j];
            if (!never_cap && qm >= t_cap) {
                newcap = true;
                capsum += (uint64_t)qm + 1;
                ++capcnt;
            } else if (!never_cand && qm >= t_cand) {
                is_cand = true;
            }
        }
        const uint32_t nb = __ballot_sync(0xffffffffu, newcap);
        if (lane == 0) capw[g] = nb;
        const uint32_t cb = __ballot_sync(0xffffffffu, is_cand);
        if (cb) {
            int base = 0;
            if (lane == 0) base = atomicAdd(&n_cand, __popc(cb));
            base = __shfl_sync(0xffffffffu, base, 0);
            const int p = base + __popc(cb & below);
            if (is_cand && p < kCandMax) cand[p] = (uint32_t)j;
        }
    }
    block_sum2<WARPS>(capsum, capcnt, red_a, red_b);
    int n_capped = capcnt;
    uint64_t r = nn - (uint64_t)n_capped;
    R = R0 - capsum;

    // later rounds over the candidate list (warp 0)
    if (warp == 0) {
        const int nc = n_cand;
        bool full = nc > kCandMax;
        bool grew = capcnt > 0;
        while (grew && !full) {
            // the list holds every block this round can cap iff R / r >= R0 / (2 n)
            if ((unsigned __int128)(2 * nn) * R < (unsigned __int128)r * R0) {
                full = true;
                break;
            }
            uint64_t s = 0;
            int c = 0;
            for (int i = lane; i < nc; i += 32) {
                const uint32_t j = cand[i];
                if (!((capw[j >> 5] >> (j & 31)) & 1u)) {
                    const uint64_t q = (uint64_t)qm1[j] + 1;
                    if (r * q >= R) {
                        s += q;
                        ++c;
                        atomicOr(&capw[j >> 5], 1u << (j & 31));
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                c += __shfl_xor_sync(0xffffffffu, c, o);
            }
            grew = c > 0;
            n_capped += c;
            r -= (uint64_t)c;
            R -= s;
            __syncwarp();  // this round's marks are visible to the next round's reads
        }
        if (lane == 0) {
            fin_R = R;
            fin_capped = n_capped;
            fin_full = full ? 1 : 0;
        }
    }
    __syncthreads();
    R = fin_R;
    n_capped = fin_capped;
    r = nn - (uint64_t)n_capped;
    if (fin_full) {
        // remaining rounds scan every block (the state so far is exact)
        for (;;) {
            uint64_t newsum = 0;
            int grew = 0;
            for (int g = g0; g < g1; ++g) {
                const int j = g * 32 + lane;
                const uint32_t word = capw[g];
                bool newcap = false;
                if (j < nkb && !((word >> lane) & 1u)) {
                    const uint64_t q = (uint64_t)qm1[j] + 1;
                    if (r * q >= R) {
                        newcap = true;
                        newsum += q;
                    }
                }
                const uint32_t nb = __ballot_sync(0xffffffffu, newcap);
                if (nb) {
                    if (lane == 0) capw[g] = word | nb;
                    grew += lane == 0 ? __popc(nb) : 0;
                }
            }
            block_sum2<WARPS>(newsum, grew, red_a, red_b);
            if (grew == 0) break;
            n_capped += grew;
            r = nn - (uint64_t)n_capped;
            R -= newsum;
        }
    }
    const uint32_t r32 = (uint32_t)r;  // r <= n < NKB < 2^16

    // SplitMix64 state of block j is base + j * gamma with
    // base = mix(seed) + (draw row * NKB + 1) * gamma; the draw row is the
    // global row, or under the paired design that of the even query block of
    // the pair (qb with its low bit cleared)
    // (row0 is a multiple of NQB: launches start at a head boundary)
    const int64_t drow =
        row0 + row - (design == ABSA_SAMPLING_PAIRED ? (int)(blockIdx.x % (unsigned)nqb) & 1 : 0);
    const uint64_t base = splitmix64_mix(seed) + ((uint64_t)drow * (uint64_t)nkb + 1) * kGamma;
    const uint32_t Rh = (uint32_t)(R >> 32), Rl = (uint32_t)R;
    int taken = 0;
    if (design != ABSA_SAMPLING_SYSTEMATIC) {
        // Poisson draws (own or paired counters): one taken word per group
        uint64_t state = base + (uint64_t)(g0 * 32 + lane) * kGamma;  // state of block j
        for (int g = g0; g < g1; ++g, state += 32 * kGamma) {
            const int j = g * 32 + lane;
            bool take = false;
            if (j < nkb) {
                if ((capw[g] >> lane) & 1u) {
                    take = true;
                } else {
                    const uint64_t rq = (uint64_t)r32 * qm1[j] + r32;
                    take = draw_taken(splitmix64_hi32(state), Rh, Rl, rq);
                }
            }
            const uint32_t tw = __ballot_sync(0xffffffffu, take);
            if (lane == 0) takew[g] = tw;
            taken += __popc(tw);
        }
    } else {
        // Systematic design.  Interval j is [A_j, A_j + a_j) with a_j = R on C
        // and r q_j elsewhere, A_j = sum_{i<j} a_i; the points are
        // (k + U/2^32) R.  With rho_j = A_j mod R (capped blocks add 0 mod R)
        // and F = floor(U R / 2^32), an uncapped interval (a_j < R) holds the
        // point of its own period iff rho_j <= F < rho_j + a_j and that of
        // the next period iff R + F < rho_j + a_j (comparisons of the exact
        // values U R vs multiples of 2^32 reduce to these on F).
        // Blocks go in super-groups of 256: lane l holds the 8 consecutive
        // blocks 8l..8l+7, sums them in order and one warp scan per
        // super-group gives each lane its starting rho; the 8 taken bits are
        // the lane's byte of the group's taken word.
        const uint32_t U = splitmix64_hi32(base);  // the draw of block 0 of the row
        const uint64_t F = (uint64_t)U * Rh + __umulhi(U, Rl);
        const int nsg = ngp >> 3;
        const int sg_per_warp = (nsg + kSampleWarps - 1) / kSampleWarps;
        const int s0 = warp * sg_per_warp, s1 = min(nsg, s0 + sg_per_warp);
        // a_j mod R of the lane's 8 blocks (0 when capped or past NKB) and their capped bits
        auto elems = [&](int sg, uint64_t (&e)[8], uint32_t &cb) {
            const int j0 = sg * 256 + lane * 8;
            const uint4 v0 = *reinterpret_cast<const uint4 *>(qm1 + j0);
            const uint4 v1 = *reinterpret_cast<const uint4 *>(qm1 + j0 + 4);
            const uint32_t qv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            const int valid = min(8, max(0, nkb - j0));
            cb = (capw[j0 >> 5] >> (j0 & 31)) & ((1u << valid) - 1u);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                e[i] = (i < valid && !((cb >> i) & 1u)) ? (uint64_t)r32 * qv[i] + r32 : 0;
        };
        uint64_t tot = 0;
        for (int sg = s0; sg < s1; ++sg) {
            uint64_t e[8];
            uint32_t cb;
            elems(sg, e, cb);
#pragma unroll
            for (int i = 0; i < 8; ++i) tot = addmod(tot, e[i], R);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot = addmod(tot, __shfl_xor_sync(0xffffffffu, tot, o), R);
        __syncthreads();  // earlier readers of red_a are done
        if (lane == 0) red_a[warp] = tot;
        __syncthreads();
        uint64_t carry = 0;  // rho of this warp's first block
        for (int w = 0; w < warp; ++w) carry = addmod(carry, red_a[w], R);
        uint8_t *takeb = reinterpret_cast<uint8_t *>(takew);
        for (int sg = s0; sg < s1; ++sg) {
            uint64_t e[8];
            uint32_t cb;
            elems(sg, e, cb);
            uint64_t lt = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) lt = addmod(lt, e[i], R);
            uint64_t inc = lt;  // inclusive scan of the lane totals, mod R
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint64_t y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc = addmod(inc, y, R);
            }
            uint64_t rho = addmod(carry, submod(inc, lt, R), R);
            uint32_t bits = cb;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint64_t a = e[i];
                if (a != 0 && ((rho <= F && F < rho + a) || R + F < rho + a)) bits |= 1u << i;
                rho = addmod(rho, a, R);
            }
            takeb[sg * 32 + lane] = (uint8_t)bits;  // byte lane&3 of group word sg*8 + lane/4
            carry = addmod(carry, __shfl_sync(0xffffffffu, inc, 31), R);
        }
        __syncthreads();  // taken words written by other warps
        for (int g = g0 + lane; g < g1; g += 32) taken += __popc(takew[g]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) taken += __shfl_xor_sync(0xffffffffu, taken, o);
    }
    if (lane == 0) warp_cnt[warp] = taken;
    __syncthreads();
    int pos = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kSampleWarps; ++w) {
        const int c = warp_cnt[w];
        pos += w < warp ? c : 0;
        total += c;
    }
    // ascending compaction of this warp's run (block ids only); the ids are
    // also kept in shared memory (the candidate list is no longer needed)
    // for the logarithm pass when they fit
    const bool ids_in_smem = min(total, cap) <= kCandMax;
    for (int g = g0; g < g1 && pos < cap; ++g) {
        const uint32_t tw = takew[g];
        if ((tw >> lane) & 1u) {
            const int p = pos + __popc(tw & below);
            if (p < cap) {
                idx_row[p] = g * 32 + lane;
                if (ids_in_smem) cand[p] = (uint32_t)(g * 32 + lane);
            }
        }
        pos += __popc(tw);
    }
    __syncthreads();  // the block ids written above are visible to the whole CTA
    // ln(pi) of the written entries, all lanes busy (the double-precision
    // logarithm would otherwise run for a whole warp per taken lane)
    const int written = min(total, cap);
    for (int p = tid; p < written; p += kSampleThreads) {
        const int j = ids_in_smem ? (int)cand[p] : idx_row[p];
        float lp = 0.f;
        if (!((capw[j >> 5] >> (j & 31)) & 1u))
            lp = (float)log((double)((uint64_t)r32 * qm1[j] + r32) / (double)R);
        lp_row[p] = lp;
    }
    if (tid == 0) {
        counts[row] = min(total, cap);
        r_R[2 * row] = r;
        r_R[2 * row + 1] = R;
        if (total > cap) atomicOr(status, ABSA_DEVFLAG_OVERFLOW);
    }
}

template <int WARPS>
static cudaError_t launch_sample_w(const float *scores, int64_t rows, int nkb, int64_t n,
                                   uint64_t seed, int design, int nqb, int cap, int32_t *counts,
                                   int32_t *kv_index, float *log_pi, uint64_t *r_R,
                                   int32_t *status, int64_t row0, int smem, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(absa_sample_kernel<WARPS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    absa_sample_kernel<WARPS><<<(unsigned)rows, 32 * WARPS, smem, stream>>>(
        scores, nkb, n, seed, cap, counts, kv_index, log_pi, r_R, status, row0, design, nqb);
    return cudaGetLastError();
}

cudaError_t launch_sample(const float *scores, int64_t rows, int nkb, int64_t n, uint64_t seed,
                          int design, int nqb, int cap, int32_t *counts, int32_t *kv_index,
                          float *log_pi, uint64_t *r_R, int32_t *status, int64_t row0,
                          cudaStream_t stream) {
    const int ngroups = (nkb + 31) / 32;
    const int ngp = (ngroups + 7) & ~7;
    const int smem = (ngp * 32 + 2 * ngp + kCandMax) * 4;
    // The shared score copy limits the CTAs per SM (228 KB, 1 KB reserved
    // per CTA); wider CTAs keep about 32 warps per SM when few CTAs fit.
    const int per_sm = (228 * 1024) / (smem + 1024);
    if (per_sm >= 4)
        return launch_sample_w<8>(scores, rows, nkb, n, seed, design, nqb, cap, counts, kv_index,
                                  log_pi, r_R, status, row0, smem, stream);
    if (per_sm >= 2)
        return launch_sample_w<16>(scores, rows, nkb, n, seed, design, nqb, cap, counts, kv_index,
                                   log_pi, r_R, status, row0, smem, stream);
    return launch_sample_w<32>(scores, rows, nkb, n, seed, design, nqb, cap, counts, kv_index,
                               log_pi, r_R, status, row0, smem, stream);
}

}  // namespace absa
