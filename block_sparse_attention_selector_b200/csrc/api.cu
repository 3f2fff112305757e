// api.cu -- the C ABI declared in include/absa.h: argument validation,
// workspace layout, tensor maps for the TMA loads, and kernel launches on the
// caller's stream.  No allocation, no synchronisation (except absa_plan_check).
#include <math.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "absa_kernels.cuh"

namespace absa {

// One warp waits on an mbarrier that nothing arrives at (no copy or MMA in
// flight), so the wait must give up after limit_cycles and set the flag.
__global__ void absa_wait_selftest_kernel(int32_t *status, long long limit_cycles) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    __syncthreads();
    mbar_wait_limit(&bar, 0, status, &abort_flag, limit_cycles);
}

cudaError_t launch_wait_selftest(int32_t *status, long long limit_cycles, cudaStream_t stream) {
    absa_wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_cycles);
    return cudaGetLastError();
}

}  // namespace absa

using namespace absa;

namespace {

struct Dims {
    int64_t BH;
    int nqb, nkb;
};

Dims dims_of(const absa_params *p) {
    Dims d;
    d.BH = (int64_t)p->B * p->H;
    d.nqb = (p->N + 127) / 128;
    d.nkb = (p->N + 3) / 4;
    return d;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct WsLayout {
    size_t kbar_hi, kbar_lo, mu, mu_hi, mu_lo, w, assign, part_m, part_s, lse, status, total;
};

WsLayout ws_layout(const absa_params *p) {
    const Dims dm = dims_of(p);
    const size_t d = (size_t)p->d;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~(size_t)255;
        return o;
    };
    WsLayout L;
    L.kbar_hi = take((size_t)dm.BH * dm.nkb * d * 2);
    L.kbar_lo = take((size_t)dm.BH * dm.nkb * d * 2);
    L.mu = take((size_t)dm.BH * dm.nqb * 8 * d * 4);
    L.mu_hi = take((size_t)dm.BH * dm.nqb * 8 * d * 2);
    L.mu_lo = take((size_t)dm.BH * dm.nqb * 8 * d * 2);
    L.w = take((size_t)dm.BH * dm.nqb * 8 * 4);
    L.assign = take((size_t)dm.BH * dm.nqb * 128);
    const size_t parts = (size_t)dm.BH * score_key_ranges(dm.nkb) * dm.nqb * 8 * 4;
    L.part_m = take(parts);
    L.part_s = take(parts);
    L.lse = take((size_t)dm.BH * dm.nqb * 8 * 4);
    L.status = take(sizeof(int32_t));
    L.total = off;
    return L;
}

absa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ABSA_OK : ABSA_ERR_CUDA; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2-D tensor of 16-bit elements [rows, cols] (cols fastest), box 64 x box_rows with
// 128-byte swizzle.
bool make_map_16(CUtensorMap *map, const void *base, int64_t rows, int cols, int box_rows,
                 CUtensorMapDataType dtype) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void *>(base), gdim, gstride,
              box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap *map, const void *base, int64_t rows, int cols,
                   int box_rows = 128) {
    return make_map_16(map, base, rows, cols, box_rows, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

bool make_map_f16(CUtensorMap *map, const void *base, int64_t rows, int cols) {
    return make_map_16(map, base, rows, cols, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}

// An NVTX range around one entry point (visible in Nsight timelines; costs a
// few nanoseconds when no tool is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

absa_status check_plan(const absa_params *p, const absa_plan *plan) {
    if (!plan) return ABSA_ERR_INVALID_ARG;
    const Dims dm = dims_of(p);
    if (plan->n_qblocks != dm.nqb || plan->n_kvblocks != dm.nkb || plan->capacity < 1)
        return ABSA_ERR_INVALID_ARG;
    if (!plan->counts || !plan->kv_index || !plan->log_pi || !plan->r_R || !plan->status)
        return ABSA_ERR_INVALID_ARG;
    if (!aligned16(plan->counts) || !aligned16(plan->kv_index) || !aligned16(plan->log_pi) ||
        !aligned16(plan->r_R) || (reinterpret_cast<uintptr_t>(plan->status) & 3u))
        return ABSA_ERR_INVALID_ARG;
    if ((double)dm.BH * dm.nqb * (double)plan->capacity > 9.0e15) return ABSA_ERR_INVALID_ARG;
    return ABSA_OK;
}

}  // namespace

extern "C" {

const char *absa_version(void) { return "absa 0.1.0 (sm_100a)"; }

const char *absa_status_string(absa_status s) {
    switch (s) {
        case ABSA_OK: return "ABSA_OK";
        case ABSA_ERR_INVALID_ARG: return "ABSA_ERR_INVALID_ARG";
        case ABSA_ERR_UNSUPPORTED: return "ABSA_ERR_UNSUPPORTED";
        case ABSA_ERR_WORKSPACE: return "ABSA_ERR_WORKSPACE";
        case ABSA_ERR_CUDA: return "ABSA_ERR_CUDA";
        case ABSA_ERR_PLAN_OVERFLOW: return "ABSA_ERR_PLAN_OVERFLOW";
        case ABSA_ERR_BAD_PLAN: return "ABSA_ERR_BAD_PLAN";
        case ABSA_ERR_TIMEOUT: return "ABSA_ERR_TIMEOUT";
    }
    return "ABSA_ERR_UNKNOWN";
}

absa_status absa_check_params(const absa_params *p) {
    if (!p) return ABSA_ERR_INVALID_ARG;
    if (p->B < 1 || p->H < 1 || p->N < 1 || p->d < 1) return ABSA_ERR_INVALID_ARG;
    if (p->T < 1 || p->Hg < 1 || p->Wg < 1 ||
        (int64_t)p->T * p->Hg * p->Wg != (int64_t)p->N)
        return ABSA_ERR_INVALID_ARG;
    if (p->budget_blocks < 1 || p->kmeans_iters < 1 || p->kmeans_iters > 16)
        return ABSA_ERR_INVALID_ARG;
    if (!isfinite(p->softmax_scale)) return ABSA_ERR_INVALID_ARG;
    if (p->sampling != ABSA_SAMPLING_POISSON && p->sampling != ABSA_SAMPLING_SYSTEMATIC &&
        p->sampling != ABSA_SAMPLING_PAIRED)
        return ABSA_ERR_INVALID_ARG;
    if (p->q_block != 128 || p->kv_block != 4 || p->n_clusters != 8) return ABSA_ERR_UNSUPPORTED;
    if (p->d != 64 && p->d != 128) return ABSA_ERR_UNSUPPORTED;
    const Dims dm = dims_of(p);
    // TMA row coordinates and per-CTA indices are 32-bit
    if (dm.BH * dm.nkb >= (int64_t)1 << 31 || dm.BH * dm.nqb * 8 >= (int64_t)1 << 31 ||
        dm.BH * p->N + 128 >= (int64_t)1 << 31)
        return ABSA_ERR_UNSUPPORTED;
    if (dm.nkb > kSampleMaxKvBlocks) return ABSA_ERR_UNSUPPORTED;
    return ABSA_OK;
}

int32_t absa_plan_capacity(const absa_params *p) {
    if (absa_check_params(p) != ABSA_OK) return -1;
    const int64_t nkb = dims_of(p).nkb;
    const int64_t n = p->budget_blocks;
    if (n >= nkb) return (int32_t)nkb;
    int64_t c = (int64_t)sqrt((double)(64 * n));
    while (c * c < 64 * n) ++c;  // ceil(8 sqrt(n))
    while (c > 0 && (c - 1) * (c - 1) >= 64 * n) --c;
    int64_t cap = ((n + c + 32 + 31) / 32) * 32;
    return (int32_t)(cap < nkb ? cap : nkb);
}

size_t absa_workspace_bytes(const absa_params *p) {
    if (absa_check_params(p) != ABSA_OK) return 0;
    return ws_layout(p).total;
}

}  // extern "C"

namespace {

// A run of whole heads: flattened (b, h) rows bh0 .. bh0 + nbh - 1.  Every
// stage works per head (pooling, k-means and the score softmax per head; plan
// rows and attention per (head, query block)), so a run computes exactly the
// values of those heads in a call over all of them.
struct HeadRun {
    int64_t bh0, nbh;
};

HeadRun all_heads(const absa_params *p) { return HeadRun{0, (int64_t)p->B * p->H}; }

// Workspace regions of a run of heads.
struct SelectPtrs {
    __half *kb_hi, *kb_lo, *mu_hi, *mu_lo;
    float *mu, *w, *part_m, *part_s, *lse;
    uint8_t *assign;
};

SelectPtrs select_ptrs(const absa_params *p, void *ws, HeadRun hr) {
    const WsLayout L = ws_layout(p);
    const Dims dm = dims_of(p);
    const int64_t d = p->d;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    SelectPtrs P;
    P.kb_hi = reinterpret_cast<__half *>(w8 + L.kbar_hi) + hr.bh0 * dm.nkb * d;
    P.kb_lo = reinterpret_cast<__half *>(w8 + L.kbar_lo) + hr.bh0 * dm.nkb * d;
    P.mu = reinterpret_cast<float *>(w8 + L.mu) + hr.bh0 * dm.nqb * 8 * d;
    P.mu_hi = reinterpret_cast<__half *>(w8 + L.mu_hi) + hr.bh0 * dm.nqb * 8 * d;
    P.mu_lo = reinterpret_cast<__half *>(w8 + L.mu_lo) + hr.bh0 * dm.nqb * 8 * d;
    P.w = reinterpret_cast<float *>(w8 + L.w) + hr.bh0 * dm.nqb * 8;
    P.assign = w8 + L.assign + hr.bh0 * dm.nqb * 128;
    const int64_t nkr = score_key_ranges(dm.nkb);
    P.part_m = reinterpret_cast<float *>(w8 + L.part_m) + hr.bh0 * nkr * dm.nqb * 8;
    P.part_s = reinterpret_cast<float *>(w8 + L.part_s) + hr.bh0 * nkr * dm.nqb * 8;
    P.lse = reinterpret_cast<float *>(w8 + L.lse) + hr.bh0 * dm.nqb * 8;
    return P;
}

int32_t *ws_status_word(const absa_params *p, void *ws) {
    return reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + ws_layout(p).status);
}

// Stages without argument checks (the callers check once).
// S2 + S3: pooled keys, centroids, weights and assignments into the workspace.
absa_status pool_kmeans_run(const absa_params *p, const void *q, const void *k, void *ws,
                            HeadRun hr, cudaStream_t s) {
    const Dims dm = dims_of(p);
    const int64_t d = p->d;
    const SelectPtrs P = select_ptrs(p, ws, hr);
    const auto *qh = static_cast<const __nv_bfloat16 *>(q) + hr.bh0 * p->N * d;
    const auto *kh = static_cast<const __nv_bfloat16 *>(k) + hr.bh0 * p->N * d;
    return from_cuda(launch_kmeans_pool(qh, kh, hr.nbh, p->N, dm.nqb, dm.nkb, p->d,
                                        p->kmeans_iters, P.mu, P.mu_hi, P.mu_lo, P.w, P.assign,
                                        P.kb_hi, P.kb_lo, s));
}

// S4: scores from the workspace written by pool_kmeans_run.
absa_status block_scores_run(const absa_params *p, float *scores, void *ws, int32_t *status,
                             HeadRun hr, cudaStream_t s) {
    const Dims dm = dims_of(p);
    const SelectPtrs P = select_ptrs(p, ws, hr);
    float *sh = scores + hr.bh0 * dm.nqb * (int64_t)dm.nkb;
    CUtensorMap tm_kb_hi, tm_kb_lo, tm_mu_hi;
    if (!make_map_f16(&tm_kb_hi, P.kb_hi, hr.nbh * dm.nkb, p->d) ||
        !make_map_f16(&tm_kb_lo, P.kb_lo, hr.nbh * dm.nkb, p->d) ||
        !make_map_f16(&tm_mu_hi, P.mu_hi, hr.nbh * dm.nqb * 8, p->d))
        return ABSA_ERR_CUDA;
    return from_cuda(launch_score(tm_kb_hi, tm_kb_lo, tm_mu_hi, P.w, P.part_m, P.part_s, P.lse,
                                  sh, hr.nbh, dm.nqb, dm.nkb, p->d, p->softmax_scale, status, s));
}

absa_status select_scores_run(const absa_params *p, const void *q, const void *k, float *scores,
                              void *ws, int32_t *status, HeadRun hr, cudaStream_t s) {
    absa_status st = pool_kmeans_run(p, q, k, ws, hr, s);
    return st == ABSA_OK ? block_scores_run(p, scores, ws, status, hr, s) : st;
}

absa_status sample_plan_run(const absa_params *p, const float *scores, const absa_plan *plan,
                            HeadRun hr, cudaStream_t s) {
    const Dims dm = dims_of(p);
    const int64_t row0 = hr.bh0 * dm.nqb, cap = plan->capacity;
    return from_cuda(launch_sample(scores + row0 * dm.nkb, hr.nbh * dm.nqb, dm.nkb,
                                   p->budget_blocks, p->seed,
                                   p->sampling, dm.nqb, plan->capacity,
                                   plan->counts + row0,
                                   plan->kv_index + row0 * cap, plan->log_pi + row0 * cap,
                                   plan->r_R + 2 * row0, plan->status, row0, s));
}

absa_status attention_run(const absa_params *p, const void *q, const void *k, const void *v,
                          const absa_plan *plan, void *o, int32_t *status, HeadRun hr,
                          cudaStream_t s, bool pairs = false,
                          const RemainderArgs *rem = nullptr) {
    const Dims dm = dims_of(p);
    const int64_t off = hr.bh0 * p->N * (int64_t)p->d;
    const auto *qh = static_cast<const __nv_bfloat16 *>(q) + off;
    const auto *kh = static_cast<const __nv_bfloat16 *>(k) + off;
    const auto *vh = static_cast<const __nv_bfloat16 *>(v) + off;
    auto *oh = static_cast<__nv_bfloat16 *>(o) + off;
    const bool dense = plan == nullptr;
    CUtensorMap tq, tk, tv;
    // sparse gathers: one 4-row box (one 4-token block) per 64-column region
    const int kv_box = dense ? kAttnTileKeys : 4;
    if (!make_map_bf16(&tq, qh, hr.nbh * p->N, p->d) ||
        !make_map_bf16(&tk, kh, hr.nbh * p->N, p->d, kv_box) ||
        !make_map_bf16(&tv, vh, hr.nbh * p->N, p->d, kv_box))
        return ABSA_ERR_CUDA;
    if (dense)
        return from_cuda(launch_attention(true, tq, tk, tv, kh, vh, oh, hr.nbh, p->N, dm.nqb,
                                          dm.nkb, p->d, p->softmax_scale, nullptr, nullptr,
                                          nullptr, 0, status, s));
    const int64_t row0 = hr.bh0 * dm.nqb, cap = plan->capacity;
    if (pairs)
        return from_cuda(launch_attention_pair(tq, tk, tv, oh, hr.nbh, p->N, dm.nqb, dm.nkb,
                                               p->d, p->softmax_scale, plan->counts + row0,
                                               plan->kv_index + row0 * cap,
                                               plan->log_pi + row0 * cap, plan->capacity,
                                               plan->status, s));
    return from_cuda(launch_attention(false, tq, tk, tv, kh, vh, oh, hr.nbh, p->N, dm.nqb,
                                      dm.nkb, p->d, p->softmax_scale, plan->counts + row0,
                                      plan->kv_index + row0 * cap, plan->log_pi + row0 * cap,
                                      plan->capacity, plan->status, s, rem));
}

// Workspace of the remainder attention: mean keys and values (bf16) of every
// group, then its key variance (f32) and token count (i32).
struct RemLayout {
    size_t mu, nu, gvar, gcnt, total;
    int64_t ngroups;
};
RemLayout rem_layout(const absa_params *p) {
    const Dims dm = dims_of(p);
    RemLayout L;
    L.ngroups = (dm.nkb + kRemGroupBlocks - 1) / kRemGroupBlocks;
    const size_t n = (size_t)dm.BH * L.ngroups;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~(size_t)255;
        return o;
    };
    L.mu = take(n * p->d * 2);
    L.nu = take(n * p->d * 2);
    L.gvar = take(n * 4);
    L.gcnt = take(n * 4);
    L.total = off;
    return L;
}

absa_status check_select_ws(const absa_params *p, const void *ws, size_t ws_bytes) {
    if (!ws || !aligned16(ws)) return ABSA_ERR_INVALID_ARG;
    return ws_bytes < ws_layout(p).total ? ABSA_ERR_WORKSPACE : ABSA_OK;
}

// status == nullptr: report into the workspace's status word (reset first).
absa_status select_scores_impl(const absa_params *p, const void *q, const void *k, float *scores,
                               void *ws, size_t ws_bytes, int32_t *status, void *stream) {
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!q || !k || !scores) return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(scores)) return ABSA_ERR_INVALID_ARG;
    if ((st = check_select_ws(p, ws, ws_bytes)) != ABSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!status) {
        status = ws_status_word(p, ws);
        if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return ABSA_ERR_CUDA;
    }
    return select_scores_run(p, q, k, scores, ws, status, all_heads(p), s);
}

absa_status sample_plan_impl(const absa_params *p, const float *scores, const absa_plan *plan,
                             bool reset_status, void *stream) {
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!scores || !aligned16(scores)) return ABSA_ERR_INVALID_ARG;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (reset_status) {
        cudaError_t e = cudaMemsetAsync(plan->status, 0, sizeof(int32_t), s);
        if (e != cudaSuccess) return from_cuda(e);
    }
    return sample_plan_run(p, scores, plan, all_heads(p), s);
}

// Built-in workspace of absa_select_scores_static: one copy per device for as
// long as the library is loaded.  Host code must not take its address
// directly (the name is a host-side stand-in); static_scratch() resolves the
// device address once per device.
static __device__ __align__(256) uint8_t g_static_scratch[ABSA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_static_scratch on the current device (nullptr on error).
void *static_scratch() {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) return nullptr;
        addr[dev] = ptr;
    }
    return addr[dev];
}

}  // namespace

extern "C" {

absa_status absa_select_scores_static(const absa_params *p, const void *q, const void *k,
                                      float *scores, void *stream) {
    NvtxRange range("absa_select_scores_static");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (ws_layout(p).total > ABSA_STATIC_SCRATCH_BYTES) return ABSA_ERR_WORKSPACE;
    void *ws = static_scratch();
    if (!ws) return ABSA_ERR_CUDA;
    return select_scores_impl(p, q, k, scores, ws, ABSA_STATIC_SCRATCH_BYTES, nullptr, stream);
}

absa_status absa_select_scores(const absa_params *p, const void *q, const void *k, float *scores,
                               void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("absa_select_scores");
    return select_scores_impl(p, q, k, scores, ws, ws_bytes, nullptr, stream);
}

absa_status absa_select_pool_kmeans(const absa_params *p, const void *q, const void *k, void *ws,
                                    size_t ws_bytes, void *stream) {
    NvtxRange range("absa_select_pool_kmeans");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!q || !k || !aligned16(q) || !aligned16(k)) return ABSA_ERR_INVALID_ARG;
    if ((st = check_select_ws(p, ws, ws_bytes)) != ABSA_OK) return st;
    return pool_kmeans_run(p, q, k, ws, all_heads(p), reinterpret_cast<cudaStream_t>(stream));
}

absa_status absa_select_block_scores(const absa_params *p, float *scores, void *ws,
                                     size_t ws_bytes, void *stream) {
    NvtxRange range("absa_select_block_scores");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!scores || !aligned16(scores)) return ABSA_ERR_INVALID_ARG;
    if ((st = check_select_ws(p, ws, ws_bytes)) != ABSA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t *status = ws_status_word(p, ws);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return ABSA_ERR_CUDA;
    return block_scores_run(p, scores, ws, status, all_heads(p), s);
}

absa_status absa_select_check(const absa_params *p, const void *ws, void *stream) {
    NvtxRange range("absa_select_check");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!ws) {  // the built-in array of absa_select_scores_static
        if (ws_layout(p).total > ABSA_STATIC_SCRATCH_BYTES) return ABSA_ERR_WORKSPACE;
        ws = static_scratch();
        if (!ws) return ABSA_ERR_CUDA;
    } else if (!aligned16(ws)) {
        return ABSA_ERR_INVALID_ARG;
    }
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ABSA_ERR_CUDA;
    int32_t flags = 0;
    if (cudaMemcpy(&flags, ws_status_word(p, const_cast<void *>(ws)), sizeof(flags),
                   cudaMemcpyDeviceToHost) != cudaSuccess)
        return ABSA_ERR_CUDA;
    return (flags & ABSA_DEVFLAG_TIMEOUT) ? ABSA_ERR_TIMEOUT : ABSA_OK;
}

absa_status absa_selftest_wait_timeout(int32_t *status, int64_t limit_cycles, void *stream) {
    NvtxRange range("absa_selftest_wait_timeout");
    if (!status || (reinterpret_cast<uintptr_t>(status) & 3u)) return ABSA_ERR_INVALID_ARG;
    if (limit_cycles < 1 || limit_cycles > kWaitLimitCycles) return ABSA_ERR_INVALID_ARG;
    return from_cuda(
        launch_wait_selftest(status, limit_cycles, reinterpret_cast<cudaStream_t>(stream)));
}

absa_status absa_sample_plan(const absa_params *p, const float *scores, const absa_plan *plan,
                             void *stream) {
    NvtxRange range("absa_sample_plan");
    return sample_plan_impl(p, scores, plan, true, stream);
}

absa_status absa_select_plan(const absa_params *p, const void *q, const void *k, float *scores,
                             const absa_plan *plan, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange range("absa_select_plan");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    if (cudaMemsetAsync(plan->status, 0, sizeof(int32_t),
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ABSA_ERR_CUDA;
    st = select_scores_impl(p, q, k, scores, ws, ws_bytes, plan->status, stream);
    if (st != ABSA_OK) return st;
    return sample_plan_impl(p, scores, plan, false, stream);
}

absa_status absa_sparse_attention(const absa_params *p, const void *q, const void *k,
                                  const void *v, const absa_plan *plan, void *o, void *stream) {
    NvtxRange range("absa_sparse_attention");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    if (!q || !k || !v || !o) return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return ABSA_ERR_INVALID_ARG;
    return attention_run(p, q, k, v, plan, o, plan->status, all_heads(p),
                         reinterpret_cast<cudaStream_t>(stream));
}

absa_status absa_sparse_attention_pairs(const absa_params *p, const void *q, const void *k,
                                        const void *v, const absa_plan *plan, void *o,
                                        void *stream) {
    NvtxRange range("absa_sparse_attention_pairs");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    if (!q || !k || !v || !o) return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return ABSA_ERR_INVALID_ARG;
    if (2 * (int64_t)plan->capacity > kPairUnionMax) return ABSA_ERR_UNSUPPORTED;
    return attention_run(p, q, k, v, plan, o, plan->status, all_heads(p),
                         reinterpret_cast<cudaStream_t>(stream), true);
}

size_t absa_remainder_workspace_bytes(const absa_params *p) {
    if (absa_check_params(p) != ABSA_OK) return 0;
    return rem_layout(p).total;
}

absa_status absa_remainder_attention(const absa_params *p, const void *q, const void *k,
                                     const void *v, const absa_plan *plan, void *o, void *ws,
                                     size_t ws_bytes, void *stream) {
    NvtxRange range("absa_remainder_attention");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    if (!q || !k || !v || !o || !ws) return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ws))
        return ABSA_ERR_INVALID_ARG;
    const RemLayout L = rem_layout(p);
    if (ws_bytes < L.total) return ABSA_ERR_WORKSPACE;
    const Dims dm = dims_of(p);
    const auto s = reinterpret_cast<cudaStream_t>(stream);
    auto *base = static_cast<uint8_t *>(ws);
    auto *mu = reinterpret_cast<__nv_bfloat16 *>(base + L.mu);
    auto *nu = reinterpret_cast<__nv_bfloat16 *>(base + L.nu);
    auto *gvar = reinterpret_cast<float *>(base + L.gvar);
    auto *gcnt = reinterpret_cast<int32_t *>(base + L.gcnt);
    cudaError_t e = launch_group_stats(static_cast<const __nv_bfloat16 *>(k),
                                       static_cast<const __nv_bfloat16 *>(v), dm.BH, p->N, p->d,
                                       (int)L.ngroups, mu, nu, gvar, gcnt, s);
    if (e != cudaSuccess) return from_cuda(e);
    RemainderArgs ra;
    memset(&ra, 0, sizeof(ra));
    if (!make_map_bf16(&ra.tm_mu, mu, dm.BH * L.ngroups, p->d, kAttnTileKeys) ||
        !make_map_bf16(&ra.tm_nu, nu, dm.BH * L.ngroups, p->d, kAttnTileKeys))
        return ABSA_ERR_CUDA;
    ra.gvar = gvar;
    ra.gcnt = gcnt;
    ra.ngroups = (int)L.ngroups;
    ra.var_coef = (float)(0.5 * (double)p->softmax_scale * (double)p->softmax_scale *
                          1.4426950408889634);
    return attention_run(p, q, k, v, plan, o, plan->status, all_heads(p), s, false, &ra);
}

absa_status absa_dense_reference(const absa_params *p, const void *q, const void *k,
                                 const void *v, void *o, int32_t *status, void *stream) {
    NvtxRange range("absa_dense_reference");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    if (!q || !k || !v || !o) return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return ABSA_ERR_INVALID_ARG;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return ABSA_ERR_INVALID_ARG;
    return attention_run(p, q, k, v, nullptr, o, status, all_heads(p),
                         reinterpret_cast<cudaStream_t>(stream));
}

absa_status absa_step_host(const absa_params *p, const void *q_host, const void *k_host,
                           const void *v_host, void *o_host, void *q, void *k, void *v, void *o,
                           float *scores, const absa_plan *plan, void *ws, size_t ws_bytes,
                           int32_t heads_per_run, void *stream, void *copy_in_stream,
                           void *copy_out_stream) {
    NvtxRange range("absa_step_host");
    absa_status st = absa_check_params(p);
    if (st != ABSA_OK) return st;
    st = check_plan(p, plan);
    if (st != ABSA_OK) return st;
    if (!q_host || !k_host || !v_host || !o_host || !q || !k || !v || !o || !scores || !ws)
        return ABSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(scores) ||
        !aligned16(ws))
        return ABSA_ERR_INVALID_ARG;
    if (heads_per_run < 1) return ABSA_ERR_INVALID_ARG;
    if (ws_bytes < ws_layout(p).total) return ABSA_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaStream_t s_in = copy_in_stream ? reinterpret_cast<cudaStream_t>(copy_in_stream) : s;
    cudaStream_t s_out = copy_out_stream ? reinterpret_cast<cudaStream_t>(copy_out_stream) : s;
    const int64_t BH = (int64_t)p->B * p->H;
    const size_t head_bytes = (size_t)p->N * (size_t)p->d * 2;

    std::vector<cudaEvent_t> events;
    auto event = [&](cudaEvent_t *ev) {
        if (cudaEventCreateWithFlags(ev, cudaEventDisableTiming) != cudaSuccess) return false;
        events.push_back(*ev);
        return true;
    };
    // Recorded events may be destroyed before they complete: their resources
    // are released once the device reaches them.
    auto finish = [&](absa_status r) {
        for (cudaEvent_t ev : events) cudaEventDestroy(ev);
        return r;
    };

    // copies into q/k/v start only after earlier work on `stream` (which may
    // still read those buffers) has finished
    cudaEvent_t ev;
    if (!event(&ev) || cudaEventRecord(ev, s) != cudaSuccess ||
        cudaStreamWaitEvent(s_in, ev, 0) != cudaSuccess ||
        cudaMemsetAsync(plan->status, 0, sizeof(int32_t), s) != cudaSuccess)
        return finish(ABSA_ERR_CUDA);
    for (int64_t bh0 = 0; bh0 < BH; bh0 += heads_per_run) {
        const HeadRun hr{bh0, std::min<int64_t>(heads_per_run, BH - bh0)};
        const size_t off = (size_t)bh0 * head_bytes, bytes = (size_t)hr.nbh * head_bytes;
        const void *src[3] = {q_host, k_host, v_host};
        void *dst[3] = {q, k, v};
        for (int i = 0; i < 3; ++i)
            if (cudaMemcpyAsync(static_cast<uint8_t *>(dst[i]) + off,
                                static_cast<const uint8_t *>(src[i]) + off, bytes,
                                cudaMemcpyHostToDevice, s_in) != cudaSuccess)
                return finish(ABSA_ERR_CUDA);
        if (!event(&ev) || cudaEventRecord(ev, s_in) != cudaSuccess ||
            cudaStreamWaitEvent(s, ev, 0) != cudaSuccess)
            return finish(ABSA_ERR_CUDA);
        st = select_scores_run(p, q, k, scores, ws, plan->status, hr, s);
        if (st == ABSA_OK) st = sample_plan_run(p, scores, plan, hr, s);
        if (st == ABSA_OK) st = attention_run(p, q, k, v, plan, o, plan->status, hr, s);
        if (st != ABSA_OK) return finish(st);
        if (!event(&ev) || cudaEventRecord(ev, s) != cudaSuccess ||
            cudaStreamWaitEvent(s_out, ev, 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<uint8_t *>(o_host) + off,
                            static_cast<const uint8_t *>(o) + off, bytes, cudaMemcpyDeviceToHost,
                            s_out) != cudaSuccess)
            return finish(ABSA_ERR_CUDA);
    }
    // `stream` completes after the last output copy
    if (!event(&ev) || cudaEventRecord(ev, s_out) != cudaSuccess ||
        cudaStreamWaitEvent(s, ev, 0) != cudaSuccess)
        return finish(ABSA_ERR_CUDA);
    return finish(ABSA_OK);
}

absa_status absa_plan_check(const absa_plan *plan, void *stream) {
    NvtxRange range("absa_plan_check");
    if (!plan || !plan->status) return ABSA_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return ABSA_ERR_CUDA;
    int32_t flags = 0;
    e = cudaMemcpy(&flags, plan->status, sizeof(flags), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return ABSA_ERR_CUDA;
    if (flags & ABSA_DEVFLAG_TIMEOUT) return ABSA_ERR_TIMEOUT;
    if (flags & ABSA_DEVFLAG_BAD_PLAN) return ABSA_ERR_BAD_PLAN;
    if (flags & ABSA_DEVFLAG_OVERFLOW) return ABSA_ERR_PLAN_OVERFLOW;
    return ABSA_OK;
}

}  // extern "C"
