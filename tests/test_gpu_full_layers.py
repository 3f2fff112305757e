"""Full-size layers through the whole GPU path, checked row by row against the oracle.

Wan2.1 720p (40 heads, 75600 tokens, last query block 80 valid rows) and
HunyuanVideo 720p (24 heads, 118800 tokens, last query block 16 valid rows)
run select_plan + sparse_attention in the launch configuration of the
benchmark; the density sweep runs the Wan2.1 480p layer at budgets of 1, 2, 5,
10, 25 and 100% of its 8190 key blocks.  The oracle recomputes sampled plan
rows (heads 0 and H-1; the first, a middle and the last query block):

- k-means centroids, weights and assignments bit-equal;
- scores within 1e-3 relative (+1e-9);
- the plan row the oracle samples from the GPU's own scores is bit-equal to the
  GPU's (counts, indices, r*, R*; ln pi within one fp32 ulp);
- the attention rows, computed by the oracle with the GPU's plan, within
  max-abs 1e-2 and relative L2 5e-3.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (dense_reference, params_for, select_plan,
                                                  sparse_attention, synthetic)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, SCORE_ABS, SCORE_REL, attention_errors,
                         device_bf16)

pytestmark = pytest.mark.gpu


def _ws_rows(w, ws, h, qb):
    """mu [8,d] f32, w [8] f32, assign [128] u8 of plan row (0, h, qb) from the workspace."""
    BH, d = w.B * w.H, w.d
    sizes = [BH * w.nkb * d * 2, BH * w.nkb * d * 2, BH * w.nqb * 8 * d * 4,
             BH * w.nqb * 8 * d * 2, BH * w.nqb * 8 * d * 2, BH * w.nqb * 8 * 4,
             BH * w.nqb * 128]
    offs, off = [], 0
    for n in sizes:
        offs.append(off)
        off = (off + n + 255) // 256 * 256
    row = h * w.nqb + qb
    mu = ws[offs[2] + row * 8 * d * 4: offs[2] + (row + 1) * 8 * d * 4]
    wt = ws[offs[5] + row * 8 * 4: offs[5] + (row + 1) * 8 * 4]
    asg = ws[offs[6] + row * 128: offs[6] + (row + 1) * 128]
    return (mu.cpu().numpy().view(np.float32).reshape(8, d), wt.cpu().numpy().view(np.float32),
            asg.cpu().numpy())


def _check_rows(w, q, k, v, p, plan, scores, ws, o, heads, qbs):
    scale = 1.0 / math.sqrt(w.d)
    cap = plan.capacity
    counts = plan.counts.cpu().numpy()
    for h in heads:
        kbar = oracle.pool_keys(k[0, h])
        for qb in qbs:
            m = min(128, w.N - 128 * qb)
            rows = slice(128 * qb, 128 * qb + m)
            # selector
            mu_r, w_r, as_r, _ = oracle.kmeans_block(q[0, h, rows])
            mu_g, w_g, as_g = _ws_rows(w, ws, h, qb)
            assert np.array_equal(mu_g, mu_r), (h, qb)
            assert np.array_equal(w_g, w_r), (h, qb)
            assert np.array_equal(as_g[:m].astype(np.int32), as_r), (h, qb)
            s_ref = oracle.block_scores(mu_r, w_r, kbar, scale)
            s_gpu = scores[0, h, qb].cpu().numpy()
            err = np.abs(s_gpu.astype(np.float64) - s_ref)
            assert np.all(err <= SCORE_REL * np.abs(s_ref) + SCORE_ABS), (h, qb, float(err.max()))
            # sampler, from the GPU's own scores
            row = h * w.nqb + qb
            idx, lp, taken, r, R = oracle.sample_row(s_gpu, p.budget_blocks, p.seed, row, cap)
            c = int(counts[0, h, qb])
            assert c == min(taken, cap), (h, qb)
            assert np.array_equal(plan.kv_index[0, h, qb, :c].cpu().numpy(), idx), (h, qb)
            rr = plan.r_R[0, h, qb].cpu().numpy().view(np.uint64)
            assert int(rr[0]) == r and int(rr[1]) == R, (h, qb)
            lp_g = plan.log_pi[0, h, qb, :c].cpu().numpy()
            assert np.all(np.abs(lp_g - lp) <= np.spacing(np.abs(lp).astype(np.float32))), (h, qb)
            # attention on the GPU's plan
            o_ref = oracle.sparse_attention_rows(q[0, h, rows], k[0, h], v[0, h], idx, lp, scale)
            o_gpu = o[0, h, rows].float().cpu().numpy()
            mx, rel = attention_errors(o_gpu, o_ref)
            assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (h, qb, mx, rel)


@pytest.mark.parametrize("w", [synthetic.WAN720, synthetic.HUNYUAN720], ids=lambda w: w.name)
def test_full_layer_sampled_rows(w):
    import torch

    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=w.seed)
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan, scores, ws = select_plan(p, qd, kd)
    o = sparse_attention(p, qd, kd, vd, plan)
    torch.cuda.synchronize()
    plan.check()
    assert 128 * w.nqb > w.N  # the last query block is padded
    _check_rows(w, q, k, v, p, plan, scores, ws, o, (0, w.H - 1), (0, w.nqb // 2, w.nqb - 1))


@pytest.fixture(scope="module")
def wan480():
    w = synthetic.WAN480
    q, k, v = synthetic.layer_qkv_bits(w)
    return w, q, k, v, device_bf16(q), device_bf16(k), device_bf16(v)


# budgets of the density sweep: round-half-up of 1, 2, 5, 10, 25 and 100% of 8190 blocks
@pytest.mark.parametrize("budget", [82, 164, 410, 819, 2048, 8190])
def test_density_sweep_sampled_rows(wan480, budget):
    import torch

    w, q, k, v, qd, kd, vd = wan480
    p = params_for(w, budget=budget, seed=3)
    plan, scores, ws = select_plan(p, qd, kd)
    o = sparse_attention(p, qd, kd, vd, plan)
    torch.cuda.synchronize()
    plan.check()
    mean = float(plan.counts.float().mean())
    assert abs(mean - budget) <= 0.05 * budget + 1, mean
    _check_rows(w, q, k, v, p, plan, scores, ws, o, (0, w.H - 1), (0, 127, w.nqb - 1))
    if budget >= w.nkb:  # every block, pi = 1: the sparse path is dense attention
        assert bool((plan.counts == w.nkb).all())
        o_dense = dense_reference(p, qd, kd, vd)
        assert torch.equal(o, o_dense)
