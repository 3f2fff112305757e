"""GPU HT sparse attention (K5) and dense attention (K6) against the oracle.

Fed the identical plan, the bf16 output must be within max-abs 1e-2 and
relative L2 5e-3 of the oracle's fp64 output over the valid query rows.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (AbsaError, Plan, _abi, dense_reference,
                                                  params_for, sparse_attention, synthetic)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, RAGGED64, RAGGED128, SMALL128,
                         attention_errors, device_bf16, gpu_out_f64, load_case, plan_from_oracle)

pytestmark = pytest.mark.gpu

CASES = [synthetic.TOY, RAGGED64, RAGGED128, SMALL128]


def _oracle_plan(w, q, k, seed=0, budget=None):
    s_ref, _, _, _ = oracle.select_scores(q, k)
    n = w.budget if budget is None else budget
    cap = oracle.plan_capacity(n, w.nkb)
    return oracle.sample_plan(s_ref, n, seed, cap)


def _assert_close(o_gpu, o_ref, what):
    mx, rel = attention_errors(o_gpu, o_ref)
    assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, f"{what}: max-abs {mx:.3g}, rel-L2 {rel:.3g}"


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_sparse_attention_identical_plan(w):
    q, k, v, p = load_case(w)
    ref_plan = _oracle_plan(w, q, k, seed=3)
    plan = plan_from_oracle(p, ref_plan)
    o = sparse_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan)
    plan.check()
    o_ref = oracle.sparse_attention(q, k, v, ref_plan)
    _assert_close(gpu_out_f64(o), o_ref, w.name)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_dense_reference(w):
    q, k, v, p = load_case(w)
    o = dense_reference(p, device_bf16(q), device_bf16(k), device_bf16(v))
    o_gpu = gpu_out_f64(o)
    o_ref = np.empty_like(o_gpu)
    for b in range(w.B):
        for h in range(w.H):
            o_ref[b, h] = oracle.dense_attention_rows(q[b, h], k[b, h], v[b, h], 1 / math.sqrt(w.d))
    _assert_close(o_gpu, o_ref, w.name)


@pytest.mark.parametrize("w", [synthetic.TOY, RAGGED128], ids=lambda w: w.name)
def test_full_budget_equals_dense(w):
    """At n >= NKB every pi = 1 and HT attention is dense attention."""
    q, k, v, p = load_case(w)
    ref_plan = _oracle_plan(w, q, k, budget=w.nkb)
    assert np.all(ref_plan["counts"] == w.nkb)
    plan = plan_from_oracle(params_for(w, budget=w.nkb), ref_plan)
    pd = params_for(w, budget=w.nkb)
    o_sp = gpu_out_f64(sparse_attention(pd, device_bf16(q), device_bf16(k), device_bf16(v), plan))
    o_de = gpu_out_f64(dense_reference(pd, device_bf16(q), device_bf16(k), device_bf16(v)))
    o_ref = oracle.sparse_attention(q, k, v, ref_plan)
    _assert_close(o_sp, o_ref, "sparse at 100%")
    _assert_close(o_de, o_ref, "dense")
    # both kernels accumulate the same tiles in the same order
    assert np.array_equal(o_sp, o_de)


def test_edge_rows_empty_partial_tiles_and_quarter_pi():
    """Rows with 0, 1, 31, 32, 33, 64, 65 blocks and a pi = 1/4 block (counts as four)."""
    w = SMALL128
    q, k, v, p = load_case(w)
    cap = 96
    B, H, nqb = w.B, w.H, w.nqb
    counts = np.zeros((B, H, nqb), np.int32)
    idx = np.zeros((B, H, nqb, cap), np.int32)
    lp = np.zeros((B, H, nqb, cap), np.float32)
    sizes = [0, 1, 31, 32, 33, 64, 65, 96]
    rng = np.random.default_rng(1)
    for i, (h, qb) in enumerate([(h, qb) for h in range(H) for qb in range(nqb)]):
        c = sizes[i % len(sizes)]
        counts[0, h, qb] = c
        idx[0, h, qb, :c] = np.sort(rng.choice(w.nkb, c, replace=False))
        lp[0, h, qb, :c] = np.log(rng.uniform(0.05, 1.0, c)).astype(np.float32)
        if c:
            lp[0, h, qb, 0] = np.float32(math.log(0.25))
    ref = dict(counts=counts, kv_index=idx, log_pi=lp, r_R=np.zeros((B, H, nqb, 2), np.uint64))
    plan = plan_from_oracle(p, ref)
    o = gpu_out_f64(sparse_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan))
    plan.check()
    o_ref = oracle.sparse_attention(q, k, v, ref)
    _assert_close(o, o_ref, "edge rows")
    for h in range(H):
        for qb in range(nqb):
            if counts[0, h, qb] == 0:
                assert np.all(o[0, h, 128 * qb:128 * qb + 128] == 0)


def test_bad_plan_rows_are_rejected_and_zeroed():
    import torch

    w = synthetic.TOY
    q, k, v, p = load_case(w)
    ref_plan = _oracle_plan(w, q, k)
    plan = plan_from_oracle(p, ref_plan)
    plan.counts[0, 0, 1] = plan.capacity + 1          # count above capacity
    plan.kv_index[0, 1, 2, 0] = w.nkb                 # index out of range
    o = sparse_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan)
    with pytest.raises(AbsaError) as e:
        plan.check()
    assert e.value.code == _abi.ABSA_ERR_BAD_PLAN
    o = o.float().cpu().numpy()
    assert np.all(o[0, 0, 128:256] == 0) and np.all(o[0, 1, 256:384] == 0)
    o_ref = oracle.sparse_attention(q, k, v, ref_plan)
    _assert_close(o[0, 0, :128].astype(np.float64), o_ref[0, 0, :128], "untouched row")
    del torch


def test_sparse_attention_wan480_sampled_rows():
    """Full Wan2.1-480p layer with an oracle plan (seeded log-normal scores); the
    oracle recomputes query blocks 0, 100 and the ragged last block of every head."""
    import torch

    w = synthetic.WAN480
    q, k, v, p = load_case(w)
    scores = synthetic.random_scores(w.H * w.nqb, w.nkb, 5, concentration=2.0)
    scores = scores.reshape(1, w.H, w.nqb, w.nkb)
    cap = oracle.plan_capacity(w.budget, w.nkb)
    ref_plan = oracle.sample_plan(scores, w.budget, 7, cap)
    del scores
    plan = plan_from_oracle(p, ref_plan)
    o = sparse_attention(p, device_bf16(q), device_bf16(k), device_bf16(v), plan)
    torch.cuda.synchronize()
    plan.check()
    o = o.float().cpu().numpy()
    for lo, hi in ((0, 1), (100, 101), (w.nqb - 1, w.nqb)):
        o_ref = oracle.sparse_attention(q, k, v, ref_plan, qb_range=(lo, hi))
        rows = slice(128 * lo, min(w.N, 128 * hi))
        _assert_close(o[:, :, rows].astype(np.float64), o_ref[:, :, rows], f"blocks {lo}:{hi}")
