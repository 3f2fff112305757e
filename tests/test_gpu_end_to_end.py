"""Independently built GPU plans against the oracle, and plan reuse.

Criteria (independent plans): at most 0.5% of the (query block, key block)
inclusion decisions differ, and every differing block is near its threshold:
|u_j / 2^32 - pi_ref,j| <= 2 |pi_gpu,j - pi_ref,j| + 2^-30.
Plan reuse (third paragraph of the AB-Attention techniques: the plan is
recomputed every four denoising steps): a plan is applied unchanged to the
next steps' drifted inputs and still matches the oracle fed the same plan.
"""
import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (params_for, select_plan, sparse_attention,
                                                  synthetic)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, RAGGED128, SMALL128, attention_errors,
                         device_bf16, gpu_out_f64, load_case, plan_to_numpy)

pytestmark = pytest.mark.gpu


def _pis(s_row, r, R):
    q = np.array(oracle.quantised_scores(s_row), dtype=np.float64)
    if R == 0:
        return np.ones(len(q))
    return np.where(r * q >= R, 1.0, r * q / R)


@pytest.mark.parametrize("w", [synthetic.TOY, RAGGED128, SMALL128], ids=lambda w: w.name)
def test_independent_plans_agree(w):
    q, k, v, p = load_case(w)
    p.seed = 17
    plan, s_gpu, _ = select_plan(p, device_bf16(q), device_bf16(k))
    plan.check()
    got = plan_to_numpy(plan)
    s_gpu = s_gpu.cpu().numpy()
    s_ref, _, _, _ = oracle.select_scores(q, k)
    cap = oracle.plan_capacity(w.budget, w.nkb)
    ref = oracle.sample_plan(s_ref, w.budget, 17, cap)
    total = differ = 0
    for b in range(w.B):
        for h in range(w.H):
            for qb in range(w.nqb):
                row = (b * w.H + h) * w.nqb + qb
                a = set(got["kv_index"][b, h, qb, :got["counts"][b, h, qb]].tolist())
                r = set(ref["kv_index"][b, h, qb, :ref["counts"][b, h, qb]].tolist())
                total += w.nkb
                diff = a ^ r
                differ += len(diff)
                if not diff:
                    continue
                pg = _pis(s_gpu[b, h, qb], *got["r_R"][b, h, qb].tolist())
                pr = _pis(s_ref[b, h, qb], *ref["r_R"][b, h, qb].tolist())
                for j in diff:
                    u = oracle.draw_u32(17, row * w.nkb + j) / 2.0 ** 32
                    assert abs(u - pr[j]) <= 2 * abs(pg[j] - pr[j]) + 2.0 ** -30, (b, h, qb, j)
    assert differ <= 0.005 * total, f"{differ} of {total} decisions differ"


def test_plan_reuse_over_four_steps():
    w = SMALL128
    q, k, v, p = load_case(w)
    plan, _, _ = select_plan(p, device_bf16(q), device_bf16(k))
    plan.check()
    before = plan_to_numpy(plan)
    qf = oracle.bf16_to_f32(q)
    kf = oracle.bf16_to_f32(k)
    for step in range(1, 4):
        qf, kf = synthetic.perturbation_bits(w, step, qf, kf)
        qs, ks = synthetic.to_bf16_bits(qf), synthetic.to_bf16_bits(kf)
        o = gpu_out_f64(sparse_attention(p, device_bf16(qs), device_bf16(ks), device_bf16(v), plan))
        plan.check()
        o_ref = oracle.sparse_attention(qs, ks, v, before)
        mx, rel = attention_errors(o, o_ref)
        assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (step, mx, rel)
    after = plan_to_numpy(plan)
    for key in before:
        assert np.array_equal(before[key], after[key]), key
