"""GPU SIP sampler (K4) against the oracle on identical score arrays.

Criteria: counts, kv_index (to count) and the audit pair (r*, R*) bit-equal;
log_pi within one fp32 ulp (both sides round a double logarithm to float).
"""
import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (AbsaError, Plan, _abi, make_params, sample_plan,
                                                  synthetic)
from gpu_helpers import plan_to_numpy

pytestmark = pytest.mark.gpu


def _params(nkb, rows_h, n, seed, sampling="poisson"):
    # a one-row-per-head layout: B=1, H=rows_h, N=4*nkb tokens with NQB = ceil(4 nkb / 128)
    N = 4 * nkb
    return make_params(1, rows_h, N, 128, 1, 1, N, n, seed=seed, sampling=sampling)


def _compare(p, scores, plan_gpu, cap):
    design = {_abi.ABSA_SAMPLING_POISSON: "poisson", _abi.ABSA_SAMPLING_SYSTEMATIC: "systematic",
              _abi.ABSA_SAMPLING_PAIRED: "paired"}[p.sampling]
    ref = oracle.sample_plan(scores, p.budget_blocks, p.seed, cap, design=design)
    got = plan_to_numpy(plan_gpu)
    assert np.array_equal(got["counts"], ref["counts"])
    assert np.array_equal(got["r_R"], ref["r_R"])
    rows = ref["counts"].reshape(-1)
    gi = got["kv_index"].reshape(len(rows), -1)
    ri = ref["kv_index"].reshape(len(rows), -1)
    gl = got["log_pi"].reshape(len(rows), -1)
    rl = ref["log_pi"].reshape(len(rows), -1)
    for i, c in enumerate(rows):
        assert np.array_equal(gi[i, :c], ri[i, :c]), f"row {i}"
        ulp = np.spacing(np.abs(rl[i, :c]).astype(np.float32))
        assert np.all(np.abs(gl[i, :c] - rl[i, :c]) <= ulp), f"row {i}"
    return ref


@pytest.mark.parametrize("nkb,H,n,seed", [(128, 2, 13, 0), (1000, 3, 100, 1), (8190, 2, 819, 2),
                                          (29700, 1, 2376, 3), (515, 2, 1, 4), (515, 2, 514, 5)])
def test_sampler_bit_exact_on_identical_scores(nkb, H, n, seed):
    import torch

    p = _params(nkb, H, n, seed)
    nqb = (p.N + 127) // 128
    scores = synthetic.random_scores(H * nqb, nkb, seed).reshape(1, H, nqb, nkb)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    plan.check()
    _compare(p, scores, plan, plan.capacity)


def test_sampler_on_oracle_selector_scores():
    import torch
    from block_sparse_attention_selector_b200 import params_for

    w = synthetic.TOY
    q, k, _ = synthetic.layer_qkv_bits(w)
    s_ref, _, _, _ = oracle.select_scores(q, k)
    p = params_for(w, seed=11)
    plan = sample_plan(p, torch.from_numpy(s_ref).cuda())
    plan.check()
    _compare(p, s_ref, plan, plan.capacity)


def test_dense_budget_takes_every_block():
    import torch

    p = _params(200, 1, 200, 3)
    nqb = (p.N + 127) // 128
    scores = synthetic.random_scores(nqb, 200, 3).reshape(1, 1, nqb, 200)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    plan.check()
    got = plan_to_numpy(plan)
    assert np.all(got["counts"] == 200)
    assert np.all(got["kv_index"][..., :200] == np.arange(200))
    assert np.all(got["log_pi"][..., :200] == 0)
    assert np.all(got["r_R"] == 0)


def test_overflow_is_flagged_and_prefix_kept():
    import torch

    p = _params(1000, 1, 300, 4)
    nqb = (p.N + 127) // 128
    scores = synthetic.random_scores(nqb, 1000, 4).reshape(1, 1, nqb, 1000)
    plan = Plan(p, "cuda", capacity=64)
    sample_plan(p, torch.from_numpy(scores).cuda(), plan)
    with pytest.raises(AbsaError) as e:
        plan.check()
    assert e.value.code == _abi.ABSA_ERR_PLAN_OVERFLOW
    _compare(p, scores, plan, 64)


def test_sampler_full_wan480_rows():
    """Every plan row of the Wan2.1-480p layer (10240 rows x 8190 blocks)."""
    import torch

    w = synthetic.WAN480
    p = make_params(w.B, w.H, w.N, w.d, w.T, w.Hg, w.Wg, w.budget, seed=9)
    scores = synthetic.random_scores(w.H * w.nqb, w.nkb, 9).reshape(1, w.H, w.nqb, w.nkb)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    plan.check()
    _compare(p, scores, plan, plan.capacity)


# The systematic design (exactly n blocks per row): same bar, every row of
# exactly n entries.
@pytest.mark.parametrize("nkb,H,n,seed,conc", [(128, 2, 13, 0, 3.0), (1000, 3, 100, 1, 0.3),
                                               (8190, 2, 819, 2, 3.0), (29700, 1, 2376, 3, 3.0),
                                               (515, 2, 1, 4, 3.0), (515, 2, 514, 5, 3.0),
                                               (8190, 1, 82, 6, 0.2), (18900, 1, 1512, 7, 1.0)])
def test_systematic_sampler_bit_exact_on_identical_scores(nkb, H, n, seed, conc):
    import torch

    p = _params(nkb, H, n, seed, sampling="systematic")
    nqb = (p.N + 127) // 128
    scores = synthetic.random_scores(H * nqb, nkb, seed, concentration=conc).reshape(1, H, nqb,
                                                                                     nkb)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    plan.check()
    ref = _compare(p, scores, plan, plan.capacity)
    assert np.all(ref["counts"] == n)


def test_systematic_full_layer_plan_and_attention():
    """select_plan with the systematic design on the Wan2.1 480p layer cut to 4
    heads: exactly n blocks per row, the plan bit-equal to the oracle's from
    the GPU's own scores, and sparse attention on it against the oracle on
    sampled query blocks."""
    import dataclasses
    import math

    import torch
    from block_sparse_attention_selector_b200 import params_for, select_plan, sparse_attention
    from gpu_helpers import ATTN_MAX_ABS, ATTN_REL_L2, attention_errors, device_bf16

    w = dataclasses.replace(synthetic.WAN480, H=4)
    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=9, sampling="systematic")
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan, scores, _ = select_plan(p, qd, kd)
    o = sparse_attention(p, qd, kd, vd, plan)
    plan.check()
    assert bool((plan.counts == w.budget).all())
    s = scores.cpu().numpy()
    ref = _compare(p, s, plan, plan.capacity)
    for h in (0, w.H - 1):
        for qb in (0, w.nqb // 2, w.nqb - 1):
            m = min(128, w.N - 128 * qb)
            rows = slice(128 * qb, 128 * qb + m)
            c = int(ref["counts"][0, h, qb])
            o_ref = oracle.sparse_attention_rows(q[0, h, rows], k[0, h], v[0, h],
                                                 ref["kv_index"][0, h, qb, :c],
                                                 ref["log_pi"][0, h, qb, :c], 1 / math.sqrt(w.d))
            mx, rel = attention_errors(o[0, h, rows].float().cpu().numpy(), o_ref)
            assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (h, qb, mx, rel)


# The paired design (query blocks 2p and 2p+1 share their draws): same bar, on
# layouts with an even and an odd number of query blocks per head (the last
# block of an odd head draws alone) and several heads.
@pytest.mark.parametrize("nkb,H,n,seed", [(128, 3, 13, 0), (515, 3, 40, 1), (1000, 2, 100, 2),
                                          (8190, 2, 819, 3), (515, 2, 514, 4)])
def test_paired_sampler_bit_exact_on_identical_scores(nkb, H, n, seed):
    import torch

    p = _params(nkb, H, n, seed, sampling="paired")
    nqb = (p.N + 127) // 128
    scores = synthetic.random_scores(H * nqb, nkb, seed, concentration=1.0).reshape(1, H, nqb,
                                                                                    nkb)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    plan.check()
    _compare(p, scores, plan, plan.capacity)


def test_paired_full_layer_plans_nest():
    """select_plan with the paired design on the Wan2.1 480p layer cut to 4
    heads: the plan bit-equal to the oracle's from the GPU's own scores, and
    within every query-block pair the row with the smaller pi_j takes block j
    only if its partner does."""
    import dataclasses

    import torch
    from block_sparse_attention_selector_b200 import params_for, select_plan
    from gpu_helpers import device_bf16

    w = dataclasses.replace(synthetic.WAN480, H=4)
    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=3, sampling="paired")
    plan, scores, _ = select_plan(p, device_bf16(q), device_bf16(k))
    plan.check()
    s = scores.cpu().numpy()
    ref = _compare(p, s, plan, plan.capacity)
    for h in (0, w.H - 1):
        for qb in range(0, w.nqb - 1, 18):  # every ninth pair
            takes = []
            pis = []
            for r in (qb, qb + 1):
                t = np.zeros(w.nkb, bool)
                t[ref["kv_index"][0, h, r, :ref["counts"][0, h, r]]] = True
                takes.append(t)
                capped, rr, RR, _ = oracle.pi_solve(s[0, h, r], w.budget)
                qv = np.array(oracle.quantised_scores(s[0, h, r]), dtype=object)
                pis.append(np.where(capped, RR, rr * qv))  # pi_j * R, exact integers
                pis[-1] = (pis[-1], RR)
            (a0, R0), (a1, R1) = pis
            lo0 = np.array([x * R1 <= y * R0 for x, y in zip(a0, a1)])  # pi_0j <= pi_1j
            t_lo = np.where(lo0, takes[0], takes[1])
            t_hi = np.where(lo0, takes[1], takes[0])
            assert not np.any(t_lo & ~t_hi), (h, qb)


# Rows that leave the sampler's fast path: the kernel keeps a shared list of
# the largest quantised scores (those at or above ceil(2^30 / n)) and runs the
# capping rounds on it while their threshold stays above the list's; rows whose
# scores do not sum to about 1 overflow the list (sum far above 1) or start
# below its threshold (sum far below 1), and then every round re-reads the
# whole row.  Special values exercise the quantisation: NaN, negative and
# zero scores count as q = 1, scores of 1 or more as q = 2^32.  The row
# lengths 515 and 8190 put row starts off 16-byte boundaries.
def _odd_rows(rows, nkb, seed):
    rng = np.random.default_rng([seed, 5])
    s = synthetic.random_scores(rows, nkb, seed, concentration=1.5).astype(np.float64)
    scale = np.array([1.0, 1e3, 1e-3, 7.0, 1e-6, 1.0, 0.5, 2.0])[np.arange(rows) % 8]
    s = (s * scale[:, None]).astype(np.float32)
    special = rows // 8 * 8 - 3 if rows >= 8 else rows - 1  # one row with special values
    idx = rng.choice(nkb, size=min(nkb, 12), replace=False)
    s[special, idx[:3]] = np.nan
    s[special, idx[3:6]] = -0.25
    s[special, idx[6:8]] = 0.0
    s[special, idx[8:10]] = 1.0
    s[special, idx[10:]] = 3.5
    return s


@pytest.mark.parametrize("design", ["poisson", "systematic", "paired"])
@pytest.mark.parametrize("nkb,H,n,seed", [(515, 3, 37, 21), (8190, 1, 819, 22),
                                          (29700, 1, 2376, 23)])
def test_sampler_fallback_paths_and_special_values(design, nkb, H, n, seed):
    import torch

    p = _params(nkb, H, n, seed, sampling=design)
    nqb = (p.N + 127) // 128
    scores = _odd_rows(H * nqb, nkb, seed).reshape(1, H, nqb, nkb)
    plan = sample_plan(p, torch.from_numpy(scores).cuda())
    try:
        plan.check()
    except AbsaError as e:  # rows far from normalised can overflow the capacity
        assert e.code == _abi.ABSA_ERR_PLAN_OVERFLOW
    _compare(p, scores, plan, plan.capacity)
