"""Helpers shared by the GPU parity tests: moving seeded inputs to the device,
reading the documented workspace layout, and the comparison criteria."""
import math

import numpy as np

import oracle
from block_sparse_attention_selector_b200 import Plan, params_for, synthetic

# Attention parity bar (bf16 in, fp32 accumulate): max-abs and relative L2.
ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 5e-3
# Score parity bar: |s_gpu - s_ref| <= SCORE_REL * s_ref + SCORE_ABS per element.
SCORE_REL = 1e-3
SCORE_ABS = 1e-9

RAGGED64 = synthetic.Workload("ragged_3x7x13_d64", 1, 3, 64, 3, 7, 13, 7, 2.0, 3.0, 5)
RAGGED128 = synthetic.Workload("ragged_2x9x30_d128", 2, 2, 128, 2, 9, 30, 14, 2.0, 3.0, 6)
SMALL128 = synthetic.Workload("small_4x16x32_d128", 1, 2, 128, 4, 16, 32, 51, 3.0, 4.0, 7)


def device_bf16(bits, device="cuda"):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def host_bits(t):
    import torch

    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def ws_views(w, ws):
    """Views of the workspace regions in the order include/absa.h documents."""
    import torch

    BH, d = w.B * w.H, w.d
    sizes = [("kbar_hi", BH * w.nkb * d * 2), ("kbar_lo", BH * w.nkb * d * 2),
             ("mu", BH * w.nqb * 8 * d * 4), ("mu_hi", BH * w.nqb * 8 * d * 2),
             ("mu_lo", BH * w.nqb * 8 * d * 2), ("w", BH * w.nqb * 8 * 4),
             ("assign", BH * w.nqb * 128)]
    out, off = {}, 0
    for name, n in sizes:
        out[name] = ws[off:off + n]
        off = (off + n + 255) // 256 * 256
    res = {
        "kbar_hi": out["kbar_hi"].view(torch.float16).reshape(w.B, w.H, w.nkb, d),
        "kbar_lo": out["kbar_lo"].view(torch.float16).reshape(w.B, w.H, w.nkb, d),
        "mu": out["mu"].view(torch.float32).reshape(w.B, w.H, w.nqb, 8, d),
        "mu_hi": out["mu_hi"].view(torch.float16).reshape(w.B, w.H, w.nqb, 8, d),
        "mu_lo": out["mu_lo"].view(torch.float16).reshape(w.B, w.H, w.nqb, 8, d),
        "w": out["w"].view(torch.float32).reshape(w.B, w.H, w.nqb, 8),
        "assign": out["assign"].reshape(w.B, w.H, w.nqb, 128),
    }
    halves = ("kbar_hi", "kbar_lo", "mu_hi", "mu_lo")
    return {k: v.float().cpu().numpy() if k in halves else v.cpu().numpy() for k, v in res.items()}


def plan_from_oracle(p, ref, device="cuda"):
    """A device Plan holding an oracle-built plan (identical-plan parity)."""
    import torch

    plan = Plan(p, device, capacity=ref["kv_index"].shape[-1])
    plan.counts.copy_(torch.from_numpy(ref["counts"]))
    plan.kv_index.copy_(torch.from_numpy(ref["kv_index"]))
    plan.log_pi.copy_(torch.from_numpy(ref["log_pi"]))
    plan.r_R.copy_(torch.from_numpy(ref["r_R"].view(np.int64)))
    return plan


def plan_to_numpy(plan):
    return dict(counts=plan.counts.cpu().numpy(), kv_index=plan.kv_index.cpu().numpy(),
                log_pi=plan.log_pi.cpu().numpy(),
                r_R=plan.r_R.cpu().numpy().view(np.uint64))


def valid_rows_mask(w):
    return np.ones(w.N, bool)


def attention_errors(o_gpu, o_ref):
    """(max-abs, relative L2) of a bf16 GPU output against an fp64 reference."""
    a = o_gpu.astype(np.float64)
    b = o_ref.astype(np.float64)
    diff = a - b
    return float(np.abs(diff).max()), float(np.linalg.norm(diff) / max(np.linalg.norm(b), 1e-300))


def gpu_out_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def pi_of_row(s_row, r, R, capped_check=True):
    """Inclusion probabilities of one plan row from its fp32 scores and (r, R)."""
    q = np.array(oracle.quantised_scores(s_row), dtype=object)
    if R == 0:
        return np.ones(len(q))
    pis = np.array([min(1.0, r * int(x) / R) if r * int(x) < R else 1.0 for x in q])
    return pis


def decision_diff(idx_a, idx_b):
    a, b = set(int(x) for x in idx_a), set(int(x) for x in idx_b)
    return sorted(a ^ b)


def scale_of(w):
    return 1.0 / math.sqrt(w.d)


def load_case(w):
    q, k, v = synthetic.layer_qkv_bits(w)
    return q, k, v, params_for(w)
