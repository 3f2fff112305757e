"""Pins of the oracle's ESTRA-style remainder attention.

Page: ESTRA (zot.news), summary and figure: queries and keys grouped, the
important pairs computed exactly, the rest approximated from group averages,
and a variance-calibrated mean correction of the representatives' weights.
The oracle's reading: the plan's blocks are exact, each group of 32
consecutive key blocks contributes its mean key and value with weight
(tokens left) * exp(s^2 |q|^2 var / 2).  Pins:
  - groups whose keys and values are constant: the representative is exact,
    so the result is dense attention for any plan (empty, partial, full, a
    ragged last group and block);
  - a plan holding every block: no remainder, dense attention on any data;
  - Gaussian keys within each group: the corrected representative tracks
    dense attention, and closer than the same representatives without the
    correction (which pins the sign and the factor 1/2 of the term);
  - the exact tokens and the representatives' weights cover every group
    exactly once: two groups of equal constant keys with values 0 and 1 give
    0.5 whatever the plan lists.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import synthetic

G = oracle.REMAINDER_GROUP_BLOCKS


def bits(x):
    return synthetic.to_bf16_bits(np.asarray(x, np.float64))


def f64(b):
    return oracle.bf16_to_f32(b).astype(np.float64)


def _constant_groups(rng, N, d):
    """k and v rows constant within every group of 4 * G tokens."""
    ng = (N + 4 * G - 1) // (4 * G)
    kg = rng.standard_normal((ng, d))
    vg = rng.standard_normal((ng, d))
    gid = np.arange(N) // (4 * G)
    return bits(kg[gid]), bits(vg[gid])


@pytest.mark.parametrize("N,d,seed", [(4 * G * 3, 16, 0), (4 * G * 4 + 37, 32, 1), (9 * 4 * G - 2, 16, 2)])
def test_constant_groups_give_dense_attention_for_any_plan(N, d, seed):
    rng = np.random.default_rng(seed)
    k, v = _constant_groups(rng, N, d)
    q = bits(rng.standard_normal((5, d)))
    nkb = (N + 3) // 4
    scale = 1.0 / math.sqrt(d)
    dense = oracle.dense_attention_rows(q, k, v, scale)
    plans = [np.zeros(0, np.int32), np.arange(nkb, dtype=np.int32),
             np.sort(rng.choice(nkb, nkb // 3, replace=False)).astype(np.int32),
             np.array([nkb - 1], np.int32)]
    for blocks in plans:
        o = oracle.remainder_attention_rows(q, k, v, blocks, scale)
        np.testing.assert_allclose(o, dense, rtol=1e-10, atol=1e-12)


def test_full_plan_is_dense_attention_on_any_data():
    rng = np.random.default_rng(3)
    N, d = 4 * G * 2 + 10, 16
    q, k, v = (bits(rng.standard_normal((n, d))) for n in (7, N, N))
    nkb = (N + 3) // 4
    scale = 1.0 / math.sqrt(d)
    o = oracle.remainder_attention_rows(q, k, v, np.arange(nkb, dtype=np.int32), scale)
    np.testing.assert_allclose(o, oracle.dense_attention_rows(q, k, v, scale), rtol=1e-10,
                               atol=1e-12)


@pytest.mark.parametrize("seed", [4, 5])
def test_variance_correction_tracks_gaussian_groups(seed):
    """Keys N(mu_g, sigma_g^2 I) with sigma_g from 0.1 to 0.6 across six groups,
    values constant per group (so the representatives' values are exact and
    only their weights matter), 64 query rows with s |q| about 1.  The
    correction exp(s^2 |q|^2 sigma_g^2 / 2) differs between the groups, so
    leaving it out biases every row toward the low-variance groups; with it,
    the error is the sampling noise of 128 keys per group."""
    rng = np.random.default_rng(seed)
    d, ng = 64, 6
    N = 4 * G * ng
    sig = np.linspace(0.1, 0.6, ng)
    mus = rng.standard_normal((ng, d)) * 0.15
    gid = np.arange(N) // (4 * G)
    k = bits(mus[gid] + sig[gid][:, None] * rng.standard_normal((N, d)))
    vg = np.eye(ng, d) * 3.0  # one value direction per group
    v = bits(vg[gid])
    scale = 1.0 / math.sqrt(d)
    q = bits(rng.standard_normal((64, d)))
    dense = oracle.dense_attention_rows(q, k, v, scale)
    corr = oracle.remainder_attention_rows(q, k, v, np.zeros(0, np.int32), scale)
    # the same representatives without the correction term
    kf, qf = f64(k), f64(q)
    mu_e = kf.reshape(ng, 4 * G, d).mean(axis=1)
    logits = scale * qf @ mu_e.T
    w = np.exp(logits - logits.max(axis=1, keepdims=True))
    unc = (w @ f64(v).reshape(ng, 4 * G, d)[:, 0]) / w.sum(axis=1, keepdims=True)
    e_corr, e_unc = np.abs(corr - dense), np.abs(unc - dense)
    assert e_corr.mean() < 0.3 * e_unc.mean(), (e_corr.mean(), e_unc.mean())
    assert e_corr.max() < 0.06, e_corr.max()


def test_weight_counts_the_tokens_left():
    """Two groups with the same constant keys and values 0 and 1: whatever is
    listed, the exact tokens plus the representatives' weights must cover
    each group exactly once, so every output is 0.5.  A rest weight that
    ignored the listed tokens would give 0.4 with half of group 0 listed."""
    d = 8
    N = 8 * G
    k = bits(np.ones((N, d)) * 0.25)
    v = bits(np.where(np.arange(N)[:, None] < 4 * G, 0.0, 1.0) * np.ones((1, d)))
    q = bits(np.ones((2, d)))
    scale = 1.0 / math.sqrt(d)
    for blocks in (np.zeros(0, np.int32), np.arange(G // 2, dtype=np.int32),
                   np.arange(G, 2 * G, dtype=np.int32)):
        o = oracle.remainder_attention_rows(q, k, v, blocks, scale)
        np.testing.assert_allclose(o, 0.5, atol=1e-12)


def test_repeated_entries_count_as_often_as_listed():
    """The same two constant groups (values 0 and 1, equal keys): a block of
    group 0 listed twice enters the exact part twice (8 tokens) and leaves the
    rest twice (120 tokens left), so group 0 still weighs 128 against 128 and
    the output stays 0.5; listing it 40 times empties the rest (no
    representative) and group 0 weighs 160: the output is 128 / 288."""
    d = 8
    N = 8 * G
    k = bits(np.ones((N, d)) * 0.25)
    v = bits(np.where(np.arange(N)[:, None] < 4 * G, 0.0, 1.0) * np.ones((1, d)))
    q = bits(np.ones((2, d)))
    s = 1.0 / math.sqrt(d)
    o = oracle.remainder_attention_rows(q, k, v, np.array([3, 3], np.int32), s)
    np.testing.assert_allclose(o, 0.5, atol=1e-12)
    o = oracle.remainder_attention_rows(q, k, v, np.full(40, 3, np.int32), s)
    np.testing.assert_allclose(o, 128.0 / 288.0, atol=1e-12)
