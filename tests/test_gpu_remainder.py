"""GPU ESTRA-style remainder attention (absa_remainder_attention) against the oracle.

The plan's blocks are the exact part, every group of 32 key blocks enters
through its variance-corrected representative (include/absa.h).  Fed the
same plan, the bf16 output must be within max-abs 1e-2 and relative L2 5e-3
of the oracle's fp64 output, as for the sparse attention: on oracle plans,
on rows that are empty (pure remainder), full (no remainder) or ragged, on
layouts with a short last group and a one-token last block, and on sampled
rows of the full Wan2.1 480p and HunyuanVideo 720p layers.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (AbsaError, _abi, params_for, remainder_attention,
                                                  select_plan, synthetic)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, RAGGED64, RAGGED128, SMALL128,
                         attention_errors, device_bf16, gpu_out_f64, load_case, plan_from_oracle)

pytestmark = pytest.mark.gpu

CASES = [synthetic.TOY, RAGGED64, RAGGED128, SMALL128]


def _assert_close(o_gpu, o_ref, what):
    mx, rel = attention_errors(o_gpu, o_ref)
    assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, f"{what}: max-abs {mx:.3g}, rel-L2 {rel:.3g}"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_remainder_on_oracle_plan(w):
    q, k, v, p = load_case(w)
    s_ref, _, _, _ = oracle.select_scores(q, k)
    cap = oracle.plan_capacity(w.budget, w.nkb)
    ref = oracle.sample_plan(s_ref, w.budget, 5, cap)
    plan = plan_from_oracle(p, ref)
    o = gpu_out_f64(remainder_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan))
    plan.check()
    _assert_close(o, oracle.remainder_attention(q, k, v, ref), w.name)


@pytest.mark.parametrize("w", [RAGGED64, SMALL128], ids=lambda w: w.name)
def test_remainder_empty_full_and_ragged_rows(w):
    """Rows with no block (pure remainder), every block (no remainder), one
    block, a whole group, and the last (short) group's blocks."""
    q, k, v, p = load_case(w)
    nkb = w.nkb
    cap = nkb
    B, H, nqb = w.B, w.H, w.nqb
    counts = np.zeros((B, H, nqb), np.int32)
    idx = np.zeros((B, H, nqb, cap), np.int32)
    lp = np.zeros((B, H, nqb, cap), np.float32)
    rng = np.random.default_rng(2)
    G = oracle.REMAINDER_GROUP_BLOCKS
    rows = [np.zeros(0, np.int32), np.arange(nkb, dtype=np.int32), np.array([nkb // 2], np.int32),
            np.arange(min(G, nkb), dtype=np.int32),
            np.arange((nkb - 1) // G * G, nkb, dtype=np.int32),
            np.sort(rng.choice(nkb, nkb // 4, replace=False)).astype(np.int32)]
    i = 0
    for h in range(H):
        for qb in range(nqb):
            r = rows[i % len(rows)]
            i += 1
            counts[0, h, qb] = len(r)
            idx[0, h, qb, :len(r)] = r
            lp[0, h, qb, :len(r)] = np.log(rng.uniform(0.1, 1.0, len(r)))  # ignored by the mode
    ref = dict(counts=counts, kv_index=idx, log_pi=lp, r_R=np.zeros((B, H, nqb, 2), np.uint64))
    plan = plan_from_oracle(p, ref)
    o = gpu_out_f64(remainder_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan))
    plan.check()
    _assert_close(o, oracle.remainder_attention(q, k, v, ref), w.name)


def test_remainder_bad_rows_and_short_workspace():
    import torch

    w = synthetic.TOY
    q, k, v, p = load_case(w)
    s_ref, _, _, _ = oracle.select_scores(q, k)
    ref = oracle.sample_plan(s_ref, w.budget, 1, oracle.plan_capacity(w.budget, w.nkb))
    plan = plan_from_oracle(p, ref)
    plan.kv_index[0, 1, 2, 0] = w.nkb  # an index out of range: that row is zeroed
    plan.counts[0, 0, 3] = plan.capacity + 1  # a count above capacity: zeroed as well
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    o = remainder_attention(p, qd, kd, vd, plan)
    with pytest.raises(AbsaError) as e:
        plan.check()
    assert e.value.code == _abi.ABSA_ERR_BAD_PLAN
    o = o.float().cpu().numpy()
    assert np.all(o[0, 1, 256:384] == 0) and np.all(o[0, 0, 384:512] == 0)
    short = torch.empty(_abi.absa_remainder_workspace_bytes(p) - 256, dtype=torch.uint8,
                        device="cuda")
    with pytest.raises(AbsaError) as e:
        remainder_attention(p, qd, kd, vd, plan, ws=short)
    assert e.value.code == _abi.ABSA_ERR_WORKSPACE


@pytest.mark.parametrize("w", [synthetic.WAN480, synthetic.HUNYUAN720], ids=lambda w: w.name)
def test_remainder_full_layer_sampled_rows(w):
    """The whole layer with the GPU's own plan; the oracle recomputes the first,
    a middle and the last query block of the first and last heads."""
    import torch

    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=11)
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan, _, _ = select_plan(p, qd, kd)
    o = remainder_attention(p, qd, kd, vd, plan)
    torch.cuda.synchronize()
    plan.check()
    counts = plan.counts.cpu().numpy()
    scale = 1.0 / math.sqrt(w.d)
    for h in (0, w.H - 1):
        for qb in (0, w.nqb // 2, w.nqb - 1):
            c = int(counts[0, h, qb])
            idx = plan.kv_index[0, h, qb, :c].cpu().numpy()
            m = min(128, w.N - 128 * qb)
            rows = slice(128 * qb, 128 * qb + m)
            o_ref = oracle.remainder_attention_rows(q[0, h, rows], k[0, h], v[0, h], idx, scale)
            mx, rel = attention_errors(o[0, h, rows].float().cpu().numpy(), o_ref)
            assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (h, qb, mx, rel)
