"""Pins of the oracle's IBCS selector (pooling, k-means, block score).

Page: AB-Attention summary (news.hamidun.com), "AB-Attention's three
techniques", IBCS paragraph.  Each test pins the oracle to something other
than itself: closed forms, invariants, special cases that reduce to a library
routine (scikit-learn's Lloyd k-means, scipy's softmax).
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

import oracle
from block_sparse_attention_selector_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(x):
    return synthetic.to_bf16_bits(np.asarray(x, np.float64))


# ------------------------------------------------------------------ pooling

@pytest.mark.parametrize("N", [16, 17, 18, 19, 64])
def test_pool_closed_form_integer_keys(N):
    d = 8
    t = np.arange(N)[:, None]
    e = np.arange(d)[None, :]
    k = bits(t + e)  # small integers: exact in bf16
    kbar = oracle.pool_keys(k)
    nkb = (N + 3) // 4
    assert kbar.shape == (nkb, d)
    for j in range(nkb):
        last = min(4 * j + 3, N - 1)
        # mean of consecutive integers 4j..last, plus the column offset
        expect = (4 * j + last) / 2.0 + np.arange(d)
        assert np.array_equal(kbar[j], expect)


def test_pool_uses_all_four_tokens():
    # one token of block 0 carries a spike: only block 0's mean moves, by spike/4
    k = np.zeros((8, 4))
    k[2, 1] = 8.0
    kbar = oracle.pool_keys(bits(k))
    assert kbar[0, 1] == 2.0 and np.count_nonzero(kbar) == 1


# ------------------------------------------------------------------ k-means

def test_kmeans_identical_queries_one_cluster():
    q = bits(np.tile(np.linspace(-1, 1, 16), (128, 1)))
    mu, w, assign, count = oracle.kmeans_block(q)
    assert np.all(assign == 0)
    assert w.tolist() == [1.0] + [0.0] * 7
    assert count.tolist() == [128] + [0] * 7
    x = oracle.bf16_to_f32(q[0])
    for c in range(8):  # empty clusters keep their initial centroid (= the same query)
        assert np.array_equal(mu[c], x)


@pytest.mark.parametrize("m", [128, 120, 80, 16, 9])
def test_kmeans_recovers_separated_groups_at_init_offsets(m):
    """Eight far-apart groups whose first members sit at offsets floor(c*m/8)."""
    rng = np.random.default_rng(m)
    d = 32
    centers = 50.0 * np.eye(8, d)
    starts = [(c * m) // 8 for c in range(8)]
    group = np.zeros(m, int)
    for c in range(8):
        end = starts[c + 1] if c < 7 else m
        group[starts[c]:end] = c
    x = centers[group] + 0.05 * rng.standard_normal((m, d))
    q = bits(x)
    mu, w, assign, count = oracle.kmeans_block(q)
    assert np.array_equal(assign, group)
    xf = oracle.bf16_to_f32(q).astype(np.float64)
    for c in range(8):
        members = xf[group == c]
        assert count[c] == len(members)
        assert w[c] == np.float32(len(members)) / np.float32(m)
        np.testing.assert_allclose(mu[c], members.mean(axis=0), rtol=0, atol=1e-5)
    assert abs(float(w.sum()) - 1.0) < 1e-6


def test_kmeans_empty_cluster_keeps_previous_centroid():
    # 8 copies of A then 8 of B: init offsets 0,2,..,14 give mu_0..3 = A, mu_4..7 = B;
    # ties go to the lowest index, so only clusters 0 and 4 have members.
    a = np.full(16, 0.5)
    b = np.full(16, -0.75)
    q = bits(np.vstack([np.tile(a, (8, 1)), np.tile(b, (8, 1))]))
    mu, w, assign, count = oracle.kmeans_block(q)
    assert assign.tolist() == [0] * 8 + [4] * 8
    assert w.tolist() == [0.5, 0, 0, 0, 0.5, 0, 0, 0]
    for c in range(8):
        np.testing.assert_array_equal(mu[c], a if c < 4 else b)


def _min_margin(x, centroids):
    d2 = ((x[:, None, :] - centroids[None, :, :]) ** 2).sum(-1)
    srt = np.sort(d2, axis=1)
    return float(np.min((srt[:, 1] - srt[:, 0]) / np.maximum(srt[:, 0], 1e-30)))


@pytest.mark.parametrize("iters", [1, 2, 3])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_kmeans_matches_sklearn_lloyd(iters, seed):
    """With no empty cluster, the oracle is scikit-learn's Lloyd from the same init."""
    from sklearn.cluster import KMeans

    w_ = synthetic.TOY
    qf, _, _ = synthetic.head_qkv(w_, 0, seed % 2)
    q = bits(qf[128 * seed: 128 * seed + 128])
    x = oracle.bf16_to_f32(q).astype(np.float64)
    init = x[[(c * 128) // 8 for c in range(8)]]
    mu, w, assign, count = oracle.kmeans_block(q, iters=iters)
    if np.any(count == 0):
        pytest.skip("an empty cluster (scikit-learn relocates those)")
    km = KMeans(n_clusters=8, init=init, n_init=1, max_iter=iters, tol=0.0, algorithm="lloyd")
    km.fit(x)
    np.testing.assert_allclose(mu, km.cluster_centers_, rtol=0, atol=2e-5)
    # the oracle's last assignment is the argmin against the previous centroids
    prev = init if iters == 1 else oracle.kmeans_block(q, iters=iters - 1)[0].astype(np.float64)
    assert _min_margin(x, prev) > 1e-4
    d2 = ((x[:, None, :] - prev[None, :, :]) ** 2).sum(-1)
    assert np.array_equal(assign, np.argmin(d2, axis=1))
    assert np.array_equal(count, np.bincount(assign, minlength=8))


def test_kmeans_centroid_is_member_mean_and_weights_are_shares():
    w_ = synthetic.TOY
    qf, _, _ = synthetic.head_qkv(w_, 0, 1)
    for qb in range(4):
        q = bits(qf[128 * qb: 128 * qb + 128])
        x = oracle.bf16_to_f32(q).astype(np.float64)
        mu, w, assign, count = oracle.kmeans_block(q)
        for c in range(8):
            if count[c]:
                np.testing.assert_allclose(mu[c], x[assign == c].mean(axis=0), atol=3e-6)
        np.testing.assert_array_equal(w * 128, count.astype(np.float32))


# ------------------------------------------------------------------- scores

def _random_head(seed, N=512, d=64):
    rng = np.random.default_rng(seed)
    return bits(rng.standard_normal((N, d))), bits(rng.standard_normal((N, d)))


def test_scores_sum_to_one():
    q, k = _random_head(3)
    kbar = oracle.pool_keys(k)
    for qb in range(4):
        mu, w, _, _ = oracle.kmeans_block(q[128 * qb:128 * qb + 128])
        s = oracle.block_scores(mu, w, kbar, 1 / 8)
        assert abs(s.sum() - 1.0) < 1e-12 and np.all(s > 0)


def test_scores_one_cluster_is_softmax_of_block_mean_keys():
    """All queries equal -> one cluster -> s = softmax(scale * kbar @ q) (block averaging)."""
    _, k = _random_head(4)
    qrow = np.random.default_rng(5).standard_normal(64)
    q = bits(np.tile(qrow, (128, 1)))
    mu, w, _, _ = oracle.kmeans_block(q)
    kbar = oracle.pool_keys(k)
    s = oracle.block_scores(mu, w, kbar, 0.125)
    x = oracle.bf16_to_f32(q[0]).astype(np.float64)
    expect = softmax(0.125 * (kbar @ x))
    np.testing.assert_allclose(s, expect, rtol=1e-12, atol=0)


def test_scores_weighted_mixture_of_centroid_softmaxes():
    """Two groups of 96 and 32 queries -> s = 0.75 softmax(l_A) + 0.25 softmax(l_B)."""
    rng = np.random.default_rng(6)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    rows = np.vstack([np.tile(a, (96, 1)), np.tile(b, (32, 1))])
    # put B's first member at an init offset so that B gets its own cluster
    order = np.arange(128)
    order[[16, 96]] = order[[96, 16]]
    q = bits(rows[order])
    mu, w, _, count = oracle.kmeans_block(q)
    _, k = _random_head(7)
    kbar = oracle.pool_keys(k)
    s = oracle.block_scores(mu, w, kbar, 0.125)
    xa = oracle.bf16_to_f32(bits(a)).astype(np.float64)
    xb = oracle.bf16_to_f32(bits(b)).astype(np.float64)
    expect = 0.75 * softmax(0.125 * kbar @ xa) + 0.25 * softmax(0.125 * kbar @ xb)
    np.testing.assert_allclose(s, expect, rtol=1e-12, atol=0)


def test_scores_scale_is_applied_to_logits():
    q, k = _random_head(8)
    kbar = oracle.pool_keys(k)
    mu, w, _, _ = oracle.kmeans_block(q[:128])
    s0 = oracle.block_scores(mu, w, kbar, 0.0)
    np.testing.assert_allclose(s0, np.full(len(s0), 1.0 / len(s0)), rtol=1e-12)


def test_whole_layer_selector_matches_per_block_pieces():
    w_ = synthetic.TOY
    q, k, _ = synthetic.layer_qkv_bits(w_)
    scores, mu, w, assign = oracle.select_scores(q, k)
    assert scores.shape == (1, 2, 4, 128)
    for h in range(2):
        kbar = oracle.pool_keys(k[0, h])
        for qb in range(4):
            mu1, w1, a1, _ = oracle.kmeans_block(q[0, h, 128 * qb:128 * qb + 128])
            np.testing.assert_array_equal(mu[0, h, qb], mu1)
            np.testing.assert_array_equal(assign[0, h, qb], a1)
            s = oracle.block_scores(mu1, w1, kbar, 1 / math.sqrt(64))
            np.testing.assert_array_equal(scores[0, h, qb], s.astype(np.float32))


def test_page_constants_fixture():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        g = json.load(f)
    assert g["query_block"]["value"] == 128
    assert g["clusters_per_block"]["value"] == 8
    assert g["kv_block_tokens"]["value"] == 4
    q, _ = _random_head(9)
    mu, w, _, _ = oracle.kmeans_block(q[:128], nc=g["clusters_per_block"]["value"])
    assert mu.shape[0] == 8 and w.shape == (8,)
