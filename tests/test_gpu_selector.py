"""GPU IBCS selector (key pooling and k-means in K2, K3 score) against the oracle.

Criteria: k-means centroids, weights and assignments bit-equal (both sides
take the decisions in fp32 with the same arithmetic order); pooled keys as an
fp16 pair hi + lo within 2^-20 of the fp64 mean; the centroids' fp16 part equal
to fp16(mu); scores within 1e-3 relative (+1e-9).
"""
import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import select_scores, synthetic
from gpu_helpers import (RAGGED64, RAGGED128, SCORE_ABS, SCORE_REL, SMALL128, device_bf16,
                         load_case, ws_views)

pytestmark = pytest.mark.gpu

CASES = [synthetic.TOY, RAGGED64, RAGGED128, SMALL128]


def _check_scores(s_gpu, s_ref):
    err = np.abs(s_gpu.astype(np.float64) - s_ref.astype(np.float64))
    bound = SCORE_REL * np.abs(s_ref.astype(np.float64)) + SCORE_ABS
    bad = err > bound
    assert not bad.any(), (
        f"{int(bad.sum())} of {bad.size} scores out of tolerance; worst ratio "
        f"{float((err / bound).max()):.3g}")


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_selector_matches_oracle(w):
    q, k, _, p = load_case(w)
    s_gpu, ws = select_scores(p, device_bf16(q), device_bf16(k))
    s_gpu = s_gpu.cpu().numpy()
    s_ref, mu_ref, w_ref, as_ref = oracle.select_scores(q, k)
    views = ws_views(w, ws)
    # k-means: identical decisions and identical fp32 centroids
    got_assign = np.where(views["assign"] == 255, -1, views["assign"].astype(np.int32))
    assert np.array_equal(got_assign, as_ref)
    assert np.array_equal(views["mu"], mu_ref)
    assert np.array_equal(views["w"], w_ref)
    # pooled keys as an fp16 pair: hi + lo within 2^-20 of the fp64 mean (the lo part
    # rounds to 2^-11 of itself, or to half the smallest fp16 subnormal, 2^-25)
    for b in range(w.B):
        for h in range(w.H):
            kbar = oracle.pool_keys(k[b, h])
            got = views["kbar_hi"][b, h].astype(np.float64) + views["kbar_lo"][b, h]
            assert np.all(np.abs(got - kbar) <= 2.0 ** -20 * np.abs(kbar) + 2.0 ** -25)
    # the centroids' fp16 part used by the score products
    assert np.array_equal(views["mu_hi"], mu_ref.astype(np.float16).astype(np.float32))
    _check_scores(s_gpu, s_ref)
    np.testing.assert_allclose(s_gpu.astype(np.float64).sum(-1), 1.0, atol=1e-4)


def test_selector_wan480_sampled_blocks():
    """Full Wan2.1-480p layer on the GPU; the oracle recomputes query blocks 0, 1, 127, 255."""
    w = synthetic.WAN480
    q, k, _, p = load_case(w)
    s_gpu, ws = select_scores(p, device_bf16(q), device_bf16(k))
    views = ws_views(w, ws)
    s_gpu = s_gpu.cpu().numpy()
    for lo, hi in ((0, 2), (127, 128), (255, 256)):
        s_ref, mu_ref, w_ref, as_ref = oracle.select_scores(q, k, qb_range=(lo, hi))
        assert np.array_equal(views["mu"][:, :, lo:hi], mu_ref[:, :, lo:hi])
        assert np.array_equal(views["w"][:, :, lo:hi], w_ref[:, :, lo:hi])
        _check_scores(s_gpu[:, :, lo:hi], s_ref[:, :, lo:hi])
    # every row of the whole layer is a distribution
    np.testing.assert_allclose(s_gpu.astype(np.float64).sum(-1), 1.0, atol=1e-4)
