"""AB-Attention block-sparse attention selector for B200 (sm_100a).

The hot path -- IBCS selector, SIP sampler and Horvitz-Thompson sparse
attention over 4-token key/value blocks, plus a dense attention kernel --
lives in libabsa.so behind the C ABI of include/absa.h.  This package binds it
with ctypes (``_abi``: the C names, raw device pointers) and offers a thin
torch-facing layer below (device memory and streams come from PyTorch; every
step of the computation runs in the library's CUDA kernels).
"""
import math

from . import _abi
from ._abi import (AbsaError, absa_check_params, absa_dense_reference, absa_params, absa_plan,
                   absa_plan_capacity, absa_plan_check, absa_sample_plan,
                   absa_select_block_scores, absa_select_check, absa_select_plan,
                   absa_select_pool_kmeans, absa_select_scores, absa_sparse_attention,
                   absa_remainder_attention, absa_remainder_workspace_bytes,
                   absa_sparse_attention_pairs, absa_step_host, absa_workspace_bytes)
from .synthetic import Workload

__all__ = [
    "AbsaError", "Plan", "Workload", "absa_check_params", "absa_dense_reference", "absa_params",
    "absa_plan", "absa_plan_capacity", "absa_plan_check", "absa_sample_plan", "absa_select_plan",
    "absa_select_block_scores", "absa_select_check", "absa_select_pool_kmeans",
    "absa_remainder_attention", "absa_remainder_workspace_bytes", "absa_select_scores",
    "absa_sparse_attention", "absa_sparse_attention_pairs", "absa_step_host",
    "absa_workspace_bytes",
    "block_scores", "dense_reference", "make_params", "pool_kmeans", "sample_plan", "select_check",
    "remainder_attention", "select_plan", "select_scores", "sparse_attention",
    "sparse_attention_pairs", "step_host",
    "workspace", "version",
]


def version():
    return _abi.version()


SAMPLING = {"poisson": _abi.ABSA_SAMPLING_POISSON, "systematic": _abi.ABSA_SAMPLING_SYSTEMATIC,
            "paired": _abi.ABSA_SAMPLING_PAIRED}


def make_params(B, H, N, d, T, Hg, Wg, budget_blocks, seed=0, softmax_scale=None,
                kmeans_iters=3, sampling="poisson"):
    """An absa_params block (q_block 128, kv_block 4, 8 clusters).

    sampling: "poisson" (independent draws), "systematic" (exactly budget_blocks
    blocks) or "paired" (Poisson draws shared by query blocks 2p and 2p+1)."""
    p = absa_params()
    p.B, p.H, p.N, p.d = int(B), int(H), int(N), int(d)
    p.T, p.Hg, p.Wg = int(T), int(Hg), int(Wg)
    p.q_block, p.kv_block, p.n_clusters = 128, 4, 8
    p.kmeans_iters = int(kmeans_iters)
    p.budget_blocks = int(budget_blocks)
    p.seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    p.softmax_scale = float(1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale)
    p.sampling = SAMPLING[sampling]
    return p


def params_for(w: Workload, seed=0, budget=None, sampling="poisson"):
    return make_params(w.B, w.H, w.N, w.d, w.T, w.Hg, w.Wg,
                       w.budget if budget is None else budget, seed, sampling=sampling)


def _stream_handle(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_bf16(*ts):
    import torch

    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v, o must be contiguous bf16 CUDA tensors [B,H,N,d]")


class Plan:
    """Device arrays of a SIP sampling plan (torch tensors) and their C view."""

    def __init__(self, p, device="cuda", capacity=None):
        import torch

        cap = absa_plan_capacity(p) if capacity is None else int(capacity)
        if cap < 1:
            raise AbsaError(_abi.ABSA_ERR_INVALID_ARG, "absa_plan_capacity")
        nqb, nkb = (p.N + 127) // 128, (p.N + 3) // 4
        rows = (p.B, p.H, nqb)
        self.capacity = cap
        self.counts = torch.zeros(rows, dtype=torch.int32, device=device)
        self.kv_index = torch.zeros(rows + (cap,), dtype=torch.int32, device=device)
        self.log_pi = torch.zeros(rows + (cap,), dtype=torch.float32, device=device)
        self.r_R = torch.zeros(rows + (2,), dtype=torch.int64, device=device)
        self.status = torch.zeros(4, dtype=torch.int32, device=device)
        self.c = absa_plan(nqb, nkb, cap, self.counts.data_ptr(), self.kv_index.data_ptr(),
                           self.log_pi.data_ptr(), self.r_R.data_ptr(), self.status.data_ptr())

    def check(self, stream=None):
        """Synchronise and raise on a device-reported error (overflow, bad plan, timeout)."""
        _abi.check(absa_plan_check(self.c, _stream_handle(stream)), "absa_plan_check")


def workspace(p, device="cuda"):
    import torch

    n = absa_workspace_bytes(p)
    if n == 0:
        raise AbsaError(_abi.ABSA_ERR_INVALID_ARG, "absa_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device)


def select_scores(p, q, k, scores=None, ws=None, stream=None):
    import torch

    _check_bf16(q, k)
    nqb, nkb = (p.N + 127) // 128, (p.N + 3) // 4
    if scores is None:
        scores = torch.empty((p.B, p.H, nqb, nkb), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(p, q.device)
    _abi.check(absa_select_scores(p, _ptr(q), _ptr(k), _ptr(scores), _ptr(ws), ws.numel(),
                                  _stream_handle(stream)), "absa_select_scores")
    return scores, ws


def pool_kmeans(p, q, k, ws, stream=None):
    """First half of select_scores: pooled keys, centroids and weights into ws."""
    _check_bf16(q, k)
    _abi.check(absa_select_pool_kmeans(p, _ptr(q), _ptr(k), _ptr(ws), ws.numel(),
                                       _stream_handle(stream)), "absa_select_pool_kmeans")
    return ws


def block_scores(p, ws, scores=None, stream=None):
    """Second half of select_scores: the block scores from the regions pool_kmeans wrote."""
    import torch

    nqb, nkb = (p.N + 127) // 128, (p.N + 3) // 4
    if scores is None:
        scores = torch.empty((p.B, p.H, nqb, nkb), dtype=torch.float32, device=ws.device)
    _abi.check(absa_select_block_scores(p, _ptr(scores), _ptr(ws), ws.numel(),
                                        _stream_handle(stream)), "absa_select_block_scores")
    return scores


def select_check(p, ws, stream=None):
    """Synchronise and raise if the last score stage on ws gave up a bounded wait."""
    _abi.check(absa_select_check(p, _ptr(ws), _stream_handle(stream)), "absa_select_check")


def sample_plan(p, scores, plan=None, stream=None):
    if plan is None:
        plan = Plan(p, scores.device)
    _abi.check(absa_sample_plan(p, _ptr(scores), plan.c, _stream_handle(stream)),
               "absa_sample_plan")
    return plan


def select_plan(p, q, k, plan=None, scores=None, ws=None, stream=None):
    import torch

    _check_bf16(q, k)
    nqb, nkb = (p.N + 127) // 128, (p.N + 3) // 4
    if plan is None:
        plan = Plan(p, q.device)
    if scores is None:
        scores = torch.empty((p.B, p.H, nqb, nkb), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(p, q.device)
    _abi.check(absa_select_plan(p, _ptr(q), _ptr(k), _ptr(scores), plan.c, _ptr(ws), ws.numel(),
                                _stream_handle(stream)), "absa_select_plan")
    return plan, scores, ws


def sparse_attention(p, q, k, v, plan, out=None, stream=None):
    import torch

    _check_bf16(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _abi.check(absa_sparse_attention(p, _ptr(q), _ptr(k), _ptr(v), plan.c, _ptr(out),
                                     _stream_handle(stream)), "absa_sparse_attention")
    return out


def sparse_attention_pairs(p, q, k, v, plan, out=None, stream=None):
    """sparse_attention with one CTA per query-block pair over the union of
    the pair's plan rows (plan capacity at most 3072)."""
    import torch

    _check_bf16(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _abi.check(absa_sparse_attention_pairs(p, _ptr(q), _ptr(k), _ptr(v), plan.c, _ptr(out),
                                           _stream_handle(stream)), "absa_sparse_attention_pairs")
    return out


def remainder_attention(p, q, k, v, plan, out=None, ws=None, stream=None):
    """ESTRA-style attention: the plan's blocks exact, every group of 32 key
    blocks through its variance-corrected representative (include/absa.h)."""
    import torch

    _check_bf16(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    nbytes = absa_remainder_workspace_bytes(p)
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _abi.check(absa_remainder_attention(p, _ptr(q), _ptr(k), _ptr(v), plan.c, _ptr(out), _ptr(ws),
                                        ws.numel(), _stream_handle(stream)),
               "absa_remainder_attention")
    return out


def dense_reference(p, q, k, v, out=None, status=None, stream=None):
    import torch

    _check_bf16(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    _abi.check(absa_dense_reference(p, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(status),
                                    _stream_handle(stream)), "absa_dense_reference")
    return out


def step_host(p, q_host, k_host, v_host, o_host, q, k, v, o, plan, scores, ws, heads_per_run=4,
              stream=None, copy_in_stream=None, copy_out_stream=None):
    """absa_step_host: the whole step on host bf16 tensors, pipelined over runs of heads.

    q_host, k_host, v_host, o_host are contiguous bf16 CPU tensors [B,H,N,d] (pin them for the
    copies to overlap the compute); q, k, v, o, plan, scores, ws are the device buffers of
    select_plan and sparse_attention.  o_host is readable once `stream` has completed.
    """
    import torch

    _check_bf16(q, k, v, o)
    for t in (q_host, k_host, v_host, o_host):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("host tensors must be contiguous bf16 CPU tensors shaped like q")
    cin = None if copy_in_stream is None else copy_in_stream.cuda_stream
    cout = None if copy_out_stream is None else copy_out_stream.cuda_stream
    _abi.check(absa_step_host(p, _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(o_host), _ptr(q),
                              _ptr(k), _ptr(v), _ptr(o), _ptr(scores), plan.c, _ptr(ws),
                              ws.numel(), int(heads_per_run), _stream_handle(stream), cin, cout),
               "absa_step_host")
    return o_host
