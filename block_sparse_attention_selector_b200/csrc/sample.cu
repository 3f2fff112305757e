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

// q - 1 as a u32 (q = max(1, floor(s 2^32)) <= 2^32).  The truncating
// conversion saturates (NaN and negatives give 0, x >= 2^32 gives 2^32 - 1,
// and no float lies in (2^32 - 256, 2^32)), so f = floor(x) clamped; then
// q - 1 = f - 1 except for f = 0 (q = 1) and the saturated f (q = 2^32).
__device__ __forceinline__ uint32_t quantise_m1(float s) {
    const uint32_t f = __float2uint_rz(s * 4294967296.0f);  // exact power-of-two scaling
    return f - ((f - 1u) < 0xFFFFFFFEu ? 1u : 0u);
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;  // SplitMix64 increment

// Upper 32 bits of the SplitMix64 output function of z.  Only the high word
// of the second product and of the last xor-shift is formed: with
// z = hi 2^32 + lo, the high word of z * c mod 2^64 is
// hi32(lo * c_lo) + lo * c_hi + hi * c_lo (mod 2^32), and the high word of
// z ^ (z >> 31) is hi ^ (hi >> 31).
// splitmix64_hi32 before its last xor-shift: u = h ^ (h >> 31), which differs
// from h in bit 0 only, so the top 31 bits of u are those of h.
__device__ __forceinline__ uint32_t splitmix64_hi32_pre(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    const uint32_t lo = (uint32_t)z, hi = (uint32_t)(z >> 32);
    return __umulhi(lo, 0x133111EBu) + lo * 0x94D049BBu + hi * 0x133111EBu;
}
__device__ __forceinline__ uint32_t splitmix64_hi32(uint64_t z) {
    const uint32_t h = splitmix64_hi32_pre(z);
    return h ^ (h >> 31);
}

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

// Shared-memory state of a plan row.
constexpr int kSampleCand = 2048;  // q - 1 of the blocks at or above the list threshold
// Iterations of 128 blocks (32 chunks of 4) in the longest row (the row start
// may sit up to 3 blocks before a 16-byte boundary).
constexpr int kSampleMaxIters = (kSampleMaxKvBlocks + 3 + 127) / 128;

// Scores of a row as 16-byte chunks: chunk c holds blocks 4c - off .. 4c - off + 3,
// where off (0..3) aligns the row start to 16 bytes; blocks outside [0, nkb)
// read as 0 and are masked by the callers.  Only the first and the last chunk
// of a row can be partial; they are read element by element, so no load
// leaves the row.
struct ScoreRow {
    const float *s;
    const float4 *s4;
    int nkb, off, nchunks;
    int full0, full1;  // chunks [full0, full1) hold 4 blocks of the row each

    __device__ ScoreRow(const float *row, int nkb_) : s(row), nkb(nkb_) {
        off = (int)((reinterpret_cast<uintptr_t>(row) >> 2) & 3u);
        s4 = reinterpret_cast<const float4 *>(row - off);
        nchunks = (nkb + off + 3) >> 2;
        full0 = off ? 1 : 0;
        full1 = (nkb + off) >> 2;
    }
    __device__ bool full(int c) const { return c >= full0 && c < full1; }
    __device__ float4 chunk(int c) const {
        const int j0 = 4 * c - off;
        if (c >= nchunks) return make_float4(0.f, 0.f, 0.f, 0.f);
        if (j0 >= 0 && j0 + 4 <= nkb) return __ldg(s4 + c);
        float4 v;
        v.x = (j0 >= 0 && j0 < nkb) ? __ldg(s + j0) : 0.f;
        v.y = (j0 + 1 >= 0 && j0 + 1 < nkb) ? __ldg(s + j0 + 1) : 0.f;
        v.z = (j0 + 2 >= 0 && j0 + 2 < nkb) ? __ldg(s + j0 + 2) : 0.f;
        v.w = (j0 + 3 >= 0 && j0 + 3 < nkb) ? __ldg(s + j0 + 3) : 0.f;
        return v;
    }
    // bit i set iff block 4c - off + i lies in [0, nkb)
    __device__ uint32_t valid_mask(int c) const {
        const int j0 = 4 * c - off;
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) m |= (j0 + i >= 0 && j0 + i < nkb) ? 1u << i : 0u;
        return m;
    }
};

// The low 8 bits of x moved to bits 0, 4, 8, ..., 28.
__device__ __forceinline__ uint32_t spread8(uint32_t x) {
    x &= 0xFFu;
    x = (x | (x << 12)) & 0x000F000Fu;
    x = (x | (x << 6)) & 0x03030303u;
    return (x | (x << 3)) & 0x11111111u;
}

__device__ __forceinline__ float f4_get(const float4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Warp-wide sum mod R (every lane gets it).
__device__ __forceinline__ uint64_t warp_sum_mod(uint64_t x, uint64_t R) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = addmod(x, __shfl_xor_sync(0xffffffffu, x, o), R);
    return x;
}

// One CTA per plan row (b,h,qb); the grid covers rows row0 .. row0+gridDim-1
// of the whole problem (scores and plan pointers start at row0, the draw
// counter uses the global row).
//  A  (from memory) q_j - 1 = quantised score, R0 = sum_j q_j, and the list of
//     q_j at or above t_list = ceil(2^30 / n) (for scores summing to about 1 that
//     is a quarter of the first capping threshold R0 / n, a few hundred blocks
//     on the workloads), in tiles of 4 * threads consecutive blocks.
//  -  Capping rounds of the definition: C_{t+1} = {j : r_t q_j >= R_t} with
//     r_t = n - |C_t|, R_t = R0 - sum_{C_t} q_j, from C_0 = {} until |C| stops
//     growing.  Every capped set contains the previous one, so each round is a
//     plain count and sum over the blocks that pass; a round runs on the list
//     whenever its threshold R_t / r_t is at least t_list (all passing blocks
//     are then listed), and otherwise (or if the list overflowed) over the
//     whole row from memory.  At the fixed point, j is capped iff
//     r* q_j >= R*.
//  C  (from memory again; the row is still in L2) the take decision of every
//     block: warp w walks its own contiguous segment of the row, 128 blocks
//     (a 16-byte chunk per lane) per step, and keeps four ballots of take bits
//     per step in shared memory.
//  -  Compaction: one scan of the warps' counts places each segment; the warp
//     walks its ballots again and writes its taken block ids in ascending
//     order.
//  -  ln(pi) of the written entries (their scores re-read by id), all threads
//     busy (the double-precision logarithm would otherwise run once per taken
//     lane of every warp step).
// Poisson draws are decided in fp32 first: with x = u/2^32 and the uncapped
// pi_j = r q_j / R, the block is taken iff x < pi_j.  d = x' - s' K with
// x' = x truncated to 23 bits, s' = s clamped to [0, 1] (NaN -> 0) and
// K = fl(r 2^32 / R) differs from x - pi_j by at most r/R (|q - s' 2^32| <= 1)
// plus 2^-21.7 of rounding, so |d| > r/R + 2^-20 decides exactly (a capped
// block, pi_j >= 1, always gives d < 0 or lands in the margin); the blocks
// within the margin take the exact integer test.
template <int WARPS>
__global__ void __launch_bounds__(32 * WARPS, WARPS == 8 ? 6 : 3) absa_sample_kernel(
    const float *__restrict__ scores, int nkb, int64_t n, uint64_t seed, int cap,
    int32_t *__restrict__ counts, int32_t *__restrict__ kv_index, float *__restrict__ log_pi,
    uint64_t *__restrict__ r_R, int32_t *status, int64_t row0, int design, int nqb) {
    constexpr int kThreads = 32 * WARPS;
    __shared__ uint32_t cand[kSampleCand];
    __shared__ uint4 takew[kSampleMaxIters];  // per step: ballots of take bit i of each lane
    __shared__ uint64_t red_a[WARPS];
    __shared__ int red_b[WARPS];
    __shared__ int wcnt[WARPS];
    __shared__ uint64_t wmod[WARPS];
    __shared__ int n_cand;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;
    const float *srow = scores + row * nkb;
    int32_t *idx_row = kv_index + row * cap;
    float *lp_row = log_pi + row * cap;

    if (n >= nkb) {  // dense budget: every block, pi = 1
        for (int j = tid; j < nkb && j < cap; j += kThreads) {
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

    const ScoreRow sr(srow, nkb);
    const int ntiles = (sr.nchunks + kThreads - 1) / kThreads;
    const uint64_t nn = (uint64_t)n;
    // t_list = ceil(2^30 / n) <= 2^30, compared on q - 1
    const uint64_t t_list = ((uint64_t)1 << 30) / nn + ((((uint64_t)1 << 30) % nn) ? 1 : 0);
    const uint32_t t_list_m1 = (uint32_t)(t_list - 1);

    // ---- pass A: R0 and the candidate list
    if (tid == 0) n_cand = 0;
    __syncthreads();
    uint64_t R0 = 0;
    {
        constexpr int kAhead = 4;  // tiles in flight per thread
        uint64_t qsum = 0;             // sum of q - 1 over the valid blocks
        int nvalid = 0;
        for (int t0 = 0; t0 < ntiles; t0 += kAhead) {
            float4 v[kAhead];
#pragma unroll
            for (int u = 0; u < kAhead; ++u) {
                const int c = (t0 + u) * kThreads + tid;
                v[u] = sr.full(c) ? __ldg(sr.s4 + c) : sr.chunk(c);
            }
#pragma unroll
            for (int u = 0; u < kAhead; ++u) {
                const int c = (t0 + u) * kThreads + tid;
                const uint32_t q0 = quantise_m1(v[u].x), q1 = quantise_m1(v[u].y);
                const uint32_t q2 = quantise_m1(v[u].z), q3 = quantise_m1(v[u].w);
                uint32_t qm[4] = {q0, q1, q2, q3};
                uint32_t valid = 0xFu;
                if (sr.full(c)) {  // the common case: no mask
                    qsum += ((uint64_t)q0 + q1) + ((uint64_t)q2 + q3);
                    nvalid += 4;
                } else {
                    valid = sr.valid_mask(c);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if ((valid >> i) & 1u) {
                            qsum += qm[i];
                            ++nvalid;
                        }
                }
                // rare: a listed block in this chunk
                if (max(max(q0, q1), max(q2, q3)) >= t_list_m1) {
                    int nc = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) nc += ((valid >> i) & 1u) && qm[i] >= t_list_m1;
                    int p = nc ? atomicAdd(&n_cand, nc) : 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (((valid >> i) & 1u) && qm[i] >= t_list_m1) {
                            if (p < kSampleCand) cand[p] = qm[i];
                            ++p;
                        }
                }
            }
        }
        R0 = qsum + (uint64_t)nvalid;
    }
    int dummy = 0;
    block_sum2<WARPS>(R0, dummy, red_a, red_b);  // its barriers also publish n_cand and cand
    const int nc_total = n_cand;
    const bool list_ok = nc_total <= kSampleCand;

    // ---- capping rounds
    uint64_t r = nn, R = R0;
    int n_capped = 0;
    for (;;) {
        uint64_t sum = 0;
        int c = 0;
        if (list_ok && R >= r * t_list) {
            for (int i = tid; i < nc_total; i += kThreads) {
                const uint64_t q = (uint64_t)cand[i] + 1;
                if (r * q >= R) {
                    sum += q;
                    ++c;
                }
            }
        } else {
            for (int t = 0; t < ntiles; ++t) {
                const int ch = t * kThreads + tid;
                const float4 v = sr.chunk(ch);
                const uint32_t valid = sr.valid_mask(ch);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint64_t q = (uint64_t)quantise_m1(f4_get(v, i)) + 1;
                    if (((valid >> i) & 1u) && r * q >= R) {
                        sum += q;
                        ++c;
                    }
                }
            }
        }
        block_sum2<WARPS>(sum, c, red_a, red_b);
        if (c == n_capped) break;  // the capped set stopped growing
        n_capped = c;
        r = nn - (uint64_t)c;
        R = R0 - sum;
    }
    const uint32_t r32 = (uint32_t)r;  // 1 <= r <= n < NKB < 2^16
    const uint32_t Rh = (uint32_t)(R >> 32), Rl = (uint32_t)R;

    // ---- pass C: take bits of this warp's segment
    // SplitMix64 state of block j is base + j * gamma with
    // base = mix(seed) + (draw row * NKB + 1) * gamma; the draw row is the
    // global row, or under the paired design that of the even query block of
    // the pair (qb with its low bit cleared)
    // (row0 is a multiple of NQB: launches start at a head boundary)
    const int64_t drow =
        row0 + row - (design == ABSA_SAMPLING_PAIRED ? (int)(blockIdx.x % (unsigned)nqb) & 1 : 0);
    const uint64_t base = splitmix64_mix(seed) + ((uint64_t)drow * (uint64_t)nkb + 1) * kGamma;
    const int niters = (sr.nchunks + 31) >> 5;
    const int per = (niters + WARPS - 1) / WARPS;
    const int i0 = min(niters, warp * per), i1 = min(niters, i0 + per);
    int wtaken = 0;  // taken blocks of this warp's segment
    // exact take bits of the 4 blocks of chunk c (capped, or the exact draw)
    auto exact_bits = [&](const float4 &v, uint64_t st, uint32_t which) -> uint32_t {
        uint32_t bits = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if ((which >> i) & 1u) {
                const uint64_t rq = (uint64_t)r32 * quantise_m1(f4_get(v, i)) + r32;
                if (rq >= R || draw_taken(splitmix64_hi32(st + (uint64_t)i * kGamma), Rh, Rl, rq))
                    bits |= 1u << i;
            }
        return bits;
    };
    auto store_bits = [&](int it, uint32_t bits) {
        const uint32_t b0 = __ballot_sync(0xffffffffu, bits & 1u);
        const uint32_t b1 = __ballot_sync(0xffffffffu, bits & 2u);
        const uint32_t b2 = __ballot_sync(0xffffffffu, bits & 4u);
        const uint32_t b3 = __ballot_sync(0xffffffffu, bits & 8u);
        if (lane == 0) takew[it] = make_uint4(b0, b1, b2, b3);
        wtaken += __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3);
    };
    if (design != ABSA_SAMPLING_SYSTEMATIC) {
        const float K = (float)((double)r * 4294967296.0 / (double)R);
        const float margin = (float)((double)r / (double)R) + 0x1p-20f;
        uint64_t st = base + (uint64_t)(int64_t)(4 * (i0 * 32 + lane) - sr.off) * kGamma;
        for (int it = i0; it < i1; ++it, st += 128 * kGamma) {
            const int c = it * 32 + lane;
            const bool full = sr.full(c);
            const float4 v = full ? __ldg(sr.s4 + c) : sr.chunk(c);
            uint32_t bits = 0;
            float dmin = INFINITY;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                // x' = 1 + u / 2^32 truncated to 23 bits needs only the top bits
                // of u; taken iff x' - s' K < 1
                const uint32_t h = splitmix64_hi32_pre(st + (uint64_t)i * kGamma);
                const float x1 = __uint_as_float((h >> 9) | 0x3F800000u);
                const float sc = __saturatef(f4_get(v, i));  // clamped to [0, 1], NaN -> 0
                const float d1 = __fmaf_rn(-sc, K, x1);
                bits |= d1 < 1.0f ? 1u << i : 0u;
                dmin = fminf(dmin, fabsf(d1 - 1.0f));
            }
            const uint32_t valid = full ? 0xFu : sr.valid_mask(c);
            if (__any_sync(0xffffffffu, dmin <= margin)) {  // rare: exact test near the threshold
                uint32_t near = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t h = splitmix64_hi32_pre(st + (uint64_t)i * kGamma);
                    const float x1 = __uint_as_float((h >> 9) | 0x3F800000u);
                    const float d1 = __fmaf_rn(-__saturatef(f4_get(v, i)), K, x1);
                    near |= fabsf(d1 - 1.0f) <= margin ? 1u << i : 0u;
                }
                near &= valid;
                bits = (bits & ~near) | exact_bits(v, st, near);
            }
            store_bits(it, bits & valid);
        }
    } else {
        // Systematic design.  Interval j is [A_j, A_j + a_j) with a_j = R on
        // C and r q_j elsewhere, A_j = sum_{i<j} a_i; the points are
        // (k + U/2^32) R.  With rho_j = A_j mod R (capped blocks add 0 mod R)
        // and F = floor(U R / 2^32), an uncapped interval (a_j < R) holds the
        // point of its own period iff rho_j <= F < rho_j + a_j and that of the
        // next period iff R + F < rho_j + a_j (comparisons of the exact values
        // U R vs multiples of 2^32 reduce to these on F).  rho comes from the
        // segment totals (first sweep, one scan over the warps) and a warp
        // scan mod R per step (second sweep).
        const uint32_t U = splitmix64_hi32(base);  // the draw of block 0 of the row
        const uint64_t F = (uint64_t)U * Rh + __umulhi(U, Rl);
        // a_j mod R of a chunk's 4 blocks (0 when capped or outside the row)
        auto elems = [&](int c, uint64_t (&e)[4], uint32_t &capped) {
            const float4 v = sr.chunk(c);
            const uint32_t valid = sr.valid_mask(c);
            capped = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint64_t rq = (uint64_t)r32 * quantise_m1(f4_get(v, i)) + r32;
                const bool in = (valid >> i) & 1u;
                if (in && rq >= R) capped |= 1u << i;
                e[i] = (in && rq < R) ? rq : 0;
            }
        };
        uint64_t seg = 0;
        for (int it = i0; it < i1; ++it) {
            uint64_t e[4];
            uint32_t cb;
            elems(it * 32 + lane, e, cb);
            uint64_t ls = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) ls = addmod(ls, e[i], R);
            seg = addmod(seg, warp_sum_mod(ls, R), R);
        }
        if (lane == 0) wmod[warp] = seg;
        __syncthreads();
        uint64_t rho0 = 0;  // rho of this segment's first block
        for (int w = 0; w < warp; ++w) rho0 = addmod(rho0, wmod[w], R);
        for (int it = i0; it < i1; ++it) {
            uint64_t e[4];
            uint32_t bits;
            elems(it * 32 + lane, e, bits);
            uint64_t ls = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) ls = addmod(ls, e[i], R);
            uint64_t inc = ls;  // inclusive warp scan mod R
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint64_t y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc = addmod(inc, y, R);
            }
            uint64_t rho = addmod(rho0, submod(inc, ls, R), R);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint64_t a = e[i];
                if (a != 0 && ((rho <= F && F < rho + a) || R + F < rho + a)) bits |= 1u << i;
                rho = addmod(rho, a, R);
            }
            rho0 = addmod(rho0, __shfl_sync(0xffffffffu, inc, 31), R);
            store_bits(it, bits);
        }
    }

    // ---- compaction: segments in warp order, ascending blocks within each
    if (lane == 0) wcnt[warp] = wtaken;
    __syncthreads();
    int pos = 0, total = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
        const int x = wcnt[w];
        pos += w < warp ? x : 0;
        total += x;
    }
    // Lane l takes 32 consecutive blocks at a time: block-order word l % 4 of
    // step l / 4 of a group of 8 steps, interleaved from the step's 4 ballots
    // (bit 4m + i of word k is take bit i of lane 8k + m); one warp scan of
    // the words' counts places them.
    for (int g0 = i0; g0 < i1 && pos < cap; g0 += 8) {
        const int it = g0 + (lane >> 2), k8 = 8 * (lane & 3);
        uint32_t word = 0;
        if (it < i1) {
            const uint4 W = takew[it];
            word = spread8(W.x >> k8) | (spread8(W.y >> k8) << 1) | (spread8(W.z >> k8) << 2) |
                   (spread8(W.w >> k8) << 3);
        }
        const int cnt = __popc(word);
        int inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        int p = pos + inc - cnt;
        const int jb = 128 * it + 4 * k8 - sr.off;
        while (word) {
            const int b = __ffs(word) - 1;
            word &= word - 1;
            if (p < cap) idx_row[p] = jb + b;
            ++p;
        }
        pos += __shfl_sync(0xffffffffu, inc, 31);
    }
    __syncthreads();  // the kv_index entries written above are visible to the whole CTA

    // ---- ln(pi) of the written entries
    const int written = min(total, cap);
    for (int p0 = tid; p0 < written; p0 += 4 * kThreads) {  // 4 entries in flight per thread
        int id[4];
        float sv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) id[u] = p0 + u * kThreads < written ? idx_row[p0 + u * kThreads] : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) sv[u] = __ldg(srow + id[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int p = p0 + u * kThreads;
            const uint64_t rqp = (uint64_t)r32 * quantise_m1(sv[u]) + r32;
            if (p < written) lp_row[p] = rqp >= R ? 0.f : (float)log((double)rqp / (double)R);
        }
    }
    if (tid == 0) {
        counts[row] = written;
        r_R[2 * row] = r;
        r_R[2 * row + 1] = R;
        if (total > cap) atomicOr(status, ABSA_DEVFLAG_OVERFLOW);
    }
}

template <int WARPS>
static cudaError_t launch_sample_w(const float *scores, int64_t rows, int nkb, int64_t n,
                                   uint64_t seed, int design, int nqb, int cap, int32_t *counts,
                                   int32_t *kv_index, float *log_pi, uint64_t *r_R,
                                   int32_t *status, int64_t row0, cudaStream_t stream) {
    absa_sample_kernel<WARPS><<<(unsigned)rows, 32 * WARPS, 0, stream>>>(
        scores, nkb, n, seed, cap, counts, kv_index, log_pi, r_R, status, row0, design, nqb);
    return cudaGetLastError();
}

cudaError_t launch_sample(const float *scores, int64_t rows, int nkb, int64_t n, uint64_t seed,
                          int design, int nqb, int cap, int32_t *counts, int32_t *kv_index,
                          float *log_pi, uint64_t *r_R, int32_t *status, int64_t row0,
                          cudaStream_t stream) {
    // Wider CTAs for long rows keep fewer rows in flight, so that a row read by
    // the first pass is still in L2 when the draw pass reads it again.
    if (nkb >= 16384)
        return launch_sample_w<16>(scores, rows, nkb, n, seed, design, nqb, cap, counts, kv_index,
                                   log_pi, r_R, status, row0, stream);
    return launch_sample_w<8>(scores, rows, nkb, n, seed, design, nqb, cap, counts, kv_index,
                              log_pi, r_R, status, row0, stream);
}

}  // namespace absa
