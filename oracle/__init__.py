"""CPU oracle of the AB-Attention hot path (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps ``liboracle.so`` (plain C,
fp64 except the fp32 k-means; see ``absa_oracle.h``) with numpy-facing
functions.  Inputs q/k/v are bf16 bit patterns as ``numpy.uint16`` arrays.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None

_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(np.uint64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_i32 = ctypes.c_int
_u64 = ctypes.c_uint64
_dbl = ctypes.c_double


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_pool_keys.argtypes = [_u16p, _i64, _i32, _f64p]
        L.oracle_kmeans_block.argtypes = [_u16p, _i32, _i32, _i32, _i32, _f32p, _f32p, _i32p, _i32p]
        L.oracle_block_scores.argtypes = [_f32p, _f32p, _i32, _i32, _f64p, _i32, _dbl, _f64p]
        L.oracle_pi_solve.argtypes = [_f32p, _i32, _i64, _u8p, ctypes.POINTER(_u64), ctypes.POINTER(_u64)]
        L.oracle_pi_solve.restype = _i32
        L.oracle_splitmix64_mix.argtypes = [_u64]
        L.oracle_splitmix64_mix.restype = _u64
        L.oracle_draw_u32.argtypes = [_u64, _u64]
        L.oracle_draw_u32.restype = ctypes.c_uint32
        L.oracle_sample_row.argtypes = [_f32p, _i32, _i64, _u64, _u64, _i32, _i32p, _f32p,
                                        ctypes.POINTER(_u64), ctypes.POINTER(_u64)]
        L.oracle_sample_row.restype = _i32
        L.oracle_sparse_attention_rows.argtypes = [_u16p, _i32, _i32, _u16p, _u16p, _i64, _i32p,
                                                   _f32p, _i32, _dbl, _f64p]
        L.oracle_dense_attention_rows.argtypes = [_u16p, _i32, _i32, _u16p, _u16p, _i64, _dbl, _f64p]
        L.oracle_remainder_attention_rows.argtypes = [_u16p, _i32, _i32, _u16p, _u16p, _i64, _i32p,
                                                      _i32, _i32, _dbl, _f64p]
        L.oracle_ht_parts.argtypes = [_u16p, _i32, _u16p, _u16p, _i64, _i32p, _f32p, _i32, _dbl,
                                      _dbl, _f64p, ctypes.POINTER(_dbl)]
        L.oracle_select_scores.argtypes = [_i32, _i32, _i64, _i32, _i32, _i32, _dbl, _u16p, _u16p,
                                           _i32, _i32, _f32p, _f32p, _f32p, _i32p]
        L.oracle_sample_plan.argtypes = [_i32, _i32, _i32, _i32, _i64, _u64, _f32p, _i32, _i32p,
                                         _i32p, _f32p, _u64p]
        L.oracle_sample_plan.restype = _i32
        L.oracle_sample_plan_design.argtypes = L.oracle_sample_plan.argtypes + [_i32]
        L.oracle_sample_plan_design.restype = _i32
        L.oracle_systematic_take.argtypes = [_f32p, _i32, _i64, ctypes.c_uint32, _u8p,
                                             ctypes.POINTER(_u64), ctypes.POINTER(_u64)]
        L.oracle_systematic_take.restype = _i32
        L.oracle_sample_row_systematic.argtypes = L.oracle_sample_row.argtypes
        L.oracle_sample_row_systematic.restype = _i32
        L.oracle_sparse_attention.argtypes = [_i32, _i32, _i64, _i32, _dbl, _u16p, _u16p, _u16p,
                                              _i32, _i32, _i32p, _i32p, _f32p, _i32, _i32, _f64p]
        L.oracle_num_threads.restype = _i32
        _lib = L
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def bf16_to_f32(bits):
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def pool_keys(k):
    """IBCS averaged keys of one head: k [N,d] bf16 bits -> kbar [ceil(N/4),d] fp64."""
    k = _c(k, np.uint16)
    N, d = k.shape
    out = np.empty(((N + 3) // 4, d), np.float64)
    lib().oracle_pool_keys(k, N, d, out)
    return out


def kmeans_block(q, nc=8, iters=3):
    """IBCS k-means of one query block q [m,d] bf16 bits -> (mu, w, assign, count)."""
    q = _c(q, np.uint16)
    m, d = q.shape
    mu = np.empty((nc, d), np.float32)
    w = np.empty(nc, np.float32)
    assign = np.empty(m, np.int32)
    count = np.empty(nc, np.int32)
    lib().oracle_kmeans_block(q, m, d, nc, iters, mu, w, assign, count)
    return mu, w, assign, count


def block_scores(mu, w, kbar, scale):
    """IBCS score row of one query block (fp64)."""
    mu = _c(mu, np.float32)
    w = _c(w, np.float32)
    kbar = _c(kbar, np.float64)
    nc, d = mu.shape
    s = np.empty(kbar.shape[0], np.float64)
    lib().oracle_block_scores(mu, w, nc, d, kbar, kbar.shape[0], float(scale), s)
    return s


def pi_solve(s, n):
    """SIP capping solve of one fp32 score row -> (capped bool[nkb], r, R, rounds)."""
    s = _c(s, np.float32)
    capped = np.empty(s.shape[0], np.uint8)
    r = _u64()
    R = _u64()
    rounds = lib().oracle_pi_solve(s, s.shape[0], int(n), capped, ctypes.byref(r), ctypes.byref(R))
    return capped.astype(bool), int(r.value), int(R.value), int(rounds)


def quantised_scores(s):
    """q_j = max(1, floor(s_j 2^32)) as Python ints (the SIP integer scores)."""
    out = []
    for x in np.asarray(s, np.float32).tolist():
        v = x * 4294967296.0
        if not (v >= 1.0):
            out.append(1)
        elif v >= 4294967296.0:
            out.append(1 << 32)
        else:
            out.append(int(math.floor(v)))
    return out


def splitmix64_mix(z):
    return int(lib().oracle_splitmix64_mix(z & 0xFFFFFFFFFFFFFFFF))


def draw_u32(seed, ctr):
    return int(lib().oracle_draw_u32(seed & 0xFFFFFFFFFFFFFFFF, ctr & 0xFFFFFFFFFFFFFFFF))


def sample_row(s, n, seed, row, cap, design="poisson"):
    """SIP plan of one score row -> (kv_index, log_pi, taken, r, R).

    design: "poisson" (independent draws) or "systematic" (exactly n blocks)."""
    s = _c(s, np.float32)
    idx = np.zeros(cap, np.int32)
    lp = np.zeros(cap, np.float32)
    r = _u64()
    R = _u64()
    fn = {"poisson": lib().oracle_sample_row,
          "systematic": lib().oracle_sample_row_systematic}[design]
    taken = fn(s, s.shape[0], int(n), int(seed), int(row), int(cap), idx, lp, ctypes.byref(r),
               ctypes.byref(R))
    m = min(taken, cap)
    return idx[:m].copy(), lp[:m].copy(), int(taken), int(r.value), int(R.value)


def sparse_attention_rows(q, k, v, blocks, log_pi, scale):
    """HT sparse attention of query rows q [m,d] over the listed 4-token blocks (fp64 out)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    blocks = _c(blocks, np.int32)
    log_pi = _c(log_pi, np.float32)
    m, d = q.shape
    o = np.empty((m, d), np.float64)
    lib().oracle_sparse_attention_rows(q, m, d, k, v, k.shape[0], blocks, log_pi, blocks.shape[0],
                                       float(scale), o)
    return o


REMAINDER_GROUP_BLOCKS = 32  # key blocks per remainder group (128 tokens)


def remainder_attention_rows(q, k, v, blocks, scale, group_blocks=REMAINDER_GROUP_BLOCKS):
    """ESTRA-style attention of query rows q [m,d]: the listed blocks exactly,
    the rest of every group of `group_blocks` key blocks through its
    variance-corrected representative (fp64 out)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    blocks = _c(blocks, np.int32)
    m, d = q.shape
    o = np.empty((m, d), np.float64)
    lib().oracle_remainder_attention_rows(q, m, d, k, v, k.shape[0], blocks, blocks.shape[0],
                                          int(group_blocks), float(scale), o)
    return o


def remainder_attention(q, k, v, plan, scale=None, qb_range=(0, 0),
                        group_blocks=REMAINDER_GROUP_BLOCKS):
    """ESTRA-style attention over a whole layer with the plan's blocks as the
    exact part (fp64 [B,H,N,d]; rows outside qb_range are NaN)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    counts, idx = plan["counts"], plan["kv_index"]
    nqb = idx.shape[2]
    lo, hi = qb_range if qb_range != (0, 0) else (0, nqb)
    o = np.full((B, H, N, d), np.nan, np.float64)
    for b in range(B):
        for h in range(H):
            for qb in range(lo, hi):
                rows = slice(128 * qb, min(N, 128 * qb + 128))
                c = int(counts[b, h, qb])
                o[b, h, rows] = remainder_attention_rows(q[b, h, rows], k[b, h], v[b, h],
                                                         idx[b, h, qb, :c], scale, group_blocks)
    return o


def dense_attention_rows(q, k, v, scale):
    """Dense softmax attention of query rows q [m,d] over all tokens (fp64 out)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    m, d = q.shape
    o = np.empty((m, d), np.float64)
    lib().oracle_dense_attention_rows(q, m, d, k, v, k.shape[0], float(scale), o)
    return o


def ht_parts(q_row, k, v, blocks, log_pi, scale, m_ref):
    """Unnormalised HT numerator (d) and normaliser for one query row."""
    q_row = _c(q_row, np.uint16).reshape(-1)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    blocks = _c(blocks, np.int32)
    log_pi = _c(log_pi, np.float32)
    d = q_row.shape[0]
    nhat = np.empty(d, np.float64)
    dhat = _dbl()
    lib().oracle_ht_parts(q_row, d, k, v, k.shape[0], blocks, log_pi, blocks.shape[0], float(scale),
                          float(m_ref), nhat, ctypes.byref(dhat))
    return nhat, float(dhat.value)


def select_scores(q, k, nc=8, iters=3, scale=None, qb_range=(0, 0)):
    """Scores [B,H,NQB,NKB] fp32 plus (mu, w, assign) for a whole layer.

    q, k: [B,H,N,d] bf16 bits.  Only query blocks in qb_range are computed
    (0,0 = all); the other rows are left zero.
    """
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    B, H, N, d = q.shape
    nqb, nkb = (N + 127) // 128, (N + 3) // 4
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    scores = np.zeros((B, H, nqb, nkb), np.float32)
    mu = np.zeros((B, H, nqb, nc, d), np.float32)
    w = np.zeros((B, H, nqb, nc), np.float32)
    assign = np.full((B, H, nqb, 128), -1, np.int32)
    lib().oracle_select_scores(B, H, N, d, nc, iters, float(scale), q, k, int(qb_range[0]),
                               int(qb_range[1]), scores, mu, w, assign)
    return scores, mu, w, assign


def systematic_take(s, n, U):
    """Systematic design on one score row with the uniform U (u32) given:
    -> (take bool[nkb], r, R)."""
    s = _c(s, np.float32)
    take = np.zeros(s.shape[0], np.uint8)
    r = _u64()
    R = _u64()
    lib().oracle_systematic_take(s, s.shape[0], int(n), int(U) & 0xFFFFFFFF, take,
                                 ctypes.byref(r), ctypes.byref(R))
    return take.astype(bool), int(r.value), int(R.value)


def sample_plan(scores, n, seed, cap, design="poisson"):
    """SIP plan for every row of a [B,H,NQB,NKB] fp32 score array.

    design: "poisson", "systematic" or "paired" (Poisson draws shared by the
    query blocks 2p and 2p+1 of a head).  Returns dict(counts, kv_index, log_pi,
    r_R, overflow_rows).
    """
    scores = _c(scores, np.float32)
    B, H, nqb, nkb = scores.shape
    counts = np.zeros((B, H, nqb), np.int32)
    idx = np.zeros((B, H, nqb, cap), np.int32)
    lp = np.zeros((B, H, nqb, cap), np.float32)
    r_R = np.zeros((B, H, nqb, 2), np.uint64)
    ov = lib().oracle_sample_plan_design(B, H, nqb, nkb, int(n), int(seed), scores, int(cap),
                                         counts, idx, lp, r_R,
                                         {"poisson": 0, "systematic": 1, "paired": 2}[design])
    return dict(counts=counts, kv_index=idx, log_pi=lp, r_R=r_R, overflow_rows=int(ov))


def sparse_attention(q, k, v, plan, scale=None, qb_range=(0, 0)):
    """HT sparse attention over a whole layer (fp64 [B,H,N,d]; rows outside qb_range are NaN)."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    counts = _c(plan["counts"], np.int32)
    idx = _c(plan["kv_index"], np.int32)
    lp = _c(plan["log_pi"], np.float32)
    nqb, cap = idx.shape[2], idx.shape[3]
    o = np.full((B, H, N, d), np.nan, np.float64)
    lib().oracle_sparse_attention(B, H, N, d, float(scale), q, k, v, nqb, cap, counts, idx, lp,
                                  int(qb_range[0]), int(qb_range[1]), o)
    return o


def num_threads():
    return int(lib().oracle_num_threads())


def plan_capacity(n, nkb):
    """Plan row capacity: min(nkb, roundup32(n + ceil(8 sqrt n) + 32))."""
    if n >= nkb:
        return nkb
    c = math.isqrt(64 * n)
    if c * c < 64 * n:
        c += 1
    cap = ((n + c + 32 + 31) // 32) * 32
    return min(nkb, cap)


__all__ = [name for name in dir() if not name.startswith("_")]
