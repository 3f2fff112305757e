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


def _params(nkb, rows_h, n, seed):
    # a one-row-per-head layout: B=1, H=rows_h, N=4*nkb tokens with NQB = ceil(4 nkb / 128)
    N = 4 * nkb
    return make_params(1, rows_h, N, 128, 1, 1, N, n, seed=seed)


def _compare(p, scores, plan_gpu, cap):
    ref = oracle.sample_plan(scores, p.budget_blocks, p.seed, cap)
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
