"""ctypes binding of libabsa.so (the C ABI in include/absa.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels.  There is no fallback: importing this module without the built
library raises.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libabsa.so")

ABSA_OK = 0
ABSA_ERR_INVALID_ARG = 1
ABSA_ERR_UNSUPPORTED = 2
ABSA_ERR_WORKSPACE = 3
ABSA_ERR_CUDA = 4
ABSA_ERR_PLAN_OVERFLOW = 5
ABSA_ERR_BAD_PLAN = 6
ABSA_ERR_TIMEOUT = 7

ABSA_DEVFLAG_OVERFLOW = 1
ABSA_DEVFLAG_BAD_PLAN = 2
ABSA_DEVFLAG_TIMEOUT = 4

EXPORTED = (
    "absa_version", "absa_status_string", "absa_check_params", "absa_plan_capacity",
    "absa_workspace_bytes", "absa_select_scores", "absa_sample_plan", "absa_select_plan",
    "absa_sparse_attention", "absa_dense_reference", "absa_plan_check",
    "absa_select_scores_static", "absa_step_host", "absa_select_pool_kmeans",
    "absa_select_block_scores", "absa_select_check", "absa_selftest_wait_timeout",
    "absa_sparse_attention_pairs", "absa_remainder_workspace_bytes", "absa_remainder_attention",
)

ABSA_STATIC_SCRATCH_BYTES = 64 << 20
ABSA_SAMPLING_POISSON = 0
ABSA_SAMPLING_SYSTEMATIC = 1
ABSA_SAMPLING_PAIRED = 2


class absa_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
        ("T", ctypes.c_int32), ("Hg", ctypes.c_int32), ("Wg", ctypes.c_int32),
        ("q_block", ctypes.c_int32), ("kv_block", ctypes.c_int32),
        ("n_clusters", ctypes.c_int32), ("kmeans_iters", ctypes.c_int32),
        ("budget_blocks", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("softmax_scale", ctypes.c_float), ("sampling", ctypes.c_int32),
    ]


class absa_plan(ctypes.Structure):
    _fields_ = [
        ("n_qblocks", ctypes.c_int32), ("n_kvblocks", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("counts", ctypes.c_void_p), ("kv_index", ctypes.c_void_p), ("log_pi", ctypes.c_void_p),
        ("r_R", ctypes.c_void_p), ("status", ctypes.c_void_p),
    ]


class AbsaError(RuntimeError):
    def __init__(self, code, where):
        self.code = int(code)
        super().__init__(f"{where}: {status_string(code)}")


_lib = None


def lib():
    """Load libabsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m block_sparse_attention_selector_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(absa_params)
        Q = ctypes.POINTER(absa_plan)
        vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        L.absa_version.restype = ctypes.c_char_p
        L.absa_status_string.argtypes = [st]
        L.absa_status_string.restype = ctypes.c_char_p
        L.absa_check_params.argtypes = [P]
        L.absa_check_params.restype = st
        L.absa_plan_capacity.argtypes = [P]
        L.absa_plan_capacity.restype = ctypes.c_int32
        L.absa_workspace_bytes.argtypes = [P]
        L.absa_workspace_bytes.restype = sz
        L.absa_select_scores.argtypes = [P, vp, vp, vp, vp, sz, vp]
        L.absa_select_scores.restype = st
        L.absa_sample_plan.argtypes = [P, vp, Q, vp]
        L.absa_sample_plan.restype = st
        L.absa_select_plan.argtypes = [P, vp, vp, vp, Q, vp, sz, vp]
        L.absa_select_plan.restype = st
        L.absa_sparse_attention.argtypes = [P, vp, vp, vp, Q, vp, vp]
        L.absa_sparse_attention.restype = st
        if hasattr(L, "absa_remainder_attention"):
            L.absa_remainder_workspace_bytes.argtypes = [P]
            L.absa_remainder_workspace_bytes.restype = ctypes.c_size_t
            L.absa_remainder_attention.argtypes = [P, vp, vp, vp, Q, vp, vp, ctypes.c_size_t, vp]
            L.absa_remainder_attention.restype = st
        if hasattr(L, "absa_sparse_attention_pairs"):
            L.absa_sparse_attention_pairs.argtypes = [P, vp, vp, vp, Q, vp, vp]
            L.absa_sparse_attention_pairs.restype = st
        L.absa_dense_reference.argtypes = [P, vp, vp, vp, vp, vp, vp]
        L.absa_dense_reference.restype = st
        L.absa_plan_check.argtypes = [Q, vp]
        L.absa_plan_check.restype = st
        L.absa_select_scores_static.argtypes = [P, vp, vp, vp, vp]
        L.absa_select_scores_static.restype = st
        L.absa_step_host.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, Q, vp, sz,
                                     ctypes.c_int32, vp, vp, vp]
        L.absa_step_host.restype = st
        L.absa_select_pool_kmeans.argtypes = [P, vp, vp, vp, sz, vp]
        L.absa_select_pool_kmeans.restype = st
        L.absa_select_block_scores.argtypes = [P, vp, vp, sz, vp]
        L.absa_select_block_scores.restype = st
        L.absa_select_check.argtypes = [P, vp, vp]
        L.absa_select_check.restype = st
        L.absa_selftest_wait_timeout.argtypes = [vp, ctypes.c_int64, vp]
        L.absa_selftest_wait_timeout.restype = st
        _lib = L
    return _lib


def status_string(code):
    return lib().absa_status_string(int(code)).decode()


def version():
    return lib().absa_version().decode()


def check(code, where):
    if code != ABSA_OK:
        raise AbsaError(code, where)


# Thin wrappers with the C names: pointers are ints (device addresses) or None.
def absa_check_params(p):
    return lib().absa_check_params(ctypes.byref(p))


def absa_plan_capacity(p):
    return lib().absa_plan_capacity(ctypes.byref(p))


def absa_workspace_bytes(p):
    return lib().absa_workspace_bytes(ctypes.byref(p))


def absa_select_scores(p, q, k, scores, ws, ws_bytes, stream):
    return lib().absa_select_scores(ctypes.byref(p), q, k, scores, ws, ws_bytes, stream)


def absa_sample_plan(p, scores, plan, stream):
    return lib().absa_sample_plan(ctypes.byref(p), scores, ctypes.byref(plan), stream)


def absa_select_plan(p, q, k, scores, plan, ws, ws_bytes, stream):
    return lib().absa_select_plan(ctypes.byref(p), q, k, scores, ctypes.byref(plan), ws, ws_bytes,
                                  stream)


def absa_sparse_attention(p, q, k, v, plan, o, stream):
    return lib().absa_sparse_attention(ctypes.byref(p), q, k, v, ctypes.byref(plan), o, stream)


def absa_sparse_attention_pairs(p, q, k, v, plan, o, stream):
    return lib().absa_sparse_attention_pairs(ctypes.byref(p), q, k, v, ctypes.byref(plan), o,
                                             stream)


def absa_remainder_workspace_bytes(p):
    return lib().absa_remainder_workspace_bytes(ctypes.byref(p))


def absa_remainder_attention(p, q, k, v, plan, o, ws, ws_bytes, stream):
    return lib().absa_remainder_attention(ctypes.byref(p), q, k, v, ctypes.byref(plan), o, ws,
                                          ws_bytes, stream)


def absa_dense_reference(p, q, k, v, o, status, stream):
    return lib().absa_dense_reference(ctypes.byref(p), q, k, v, o, status, stream)


def absa_plan_check(plan, stream):
    return lib().absa_plan_check(ctypes.byref(plan), stream)


def absa_select_scores_static(p, q, k, scores, stream):
    """Selector scores with the library's built-in scratch (no workspace argument)."""
    return lib().absa_select_scores_static(ctypes.byref(p), q, k, scores, stream)


def absa_step_host(p, q_host, k_host, v_host, o_host, q, k, v, o, scores, plan, ws, ws_bytes,
                   heads_per_run, stream, copy_in_stream, copy_out_stream):
    return lib().absa_step_host(ctypes.byref(p), q_host, k_host, v_host, o_host, q, k, v, o,
                                scores, ctypes.byref(plan), ws, ws_bytes, heads_per_run, stream,
                                copy_in_stream, copy_out_stream)


def absa_select_pool_kmeans(p, q, k, ws, ws_bytes, stream):
    return lib().absa_select_pool_kmeans(ctypes.byref(p), q, k, ws, ws_bytes, stream)


def absa_select_block_scores(p, scores, ws, ws_bytes, stream):
    return lib().absa_select_block_scores(ctypes.byref(p), scores, ws, ws_bytes, stream)


def absa_select_check(p, ws, stream):
    """Synchronise and read the selector's status word (ws None: the built-in array)."""
    return lib().absa_select_check(ctypes.byref(p), ws, stream)


def absa_selftest_wait_timeout(status, limit_cycles, stream):
    return lib().absa_selftest_wait_timeout(status, int(limit_cycles), stream)
