"""Pins of the oracle's Horvitz-Thompson sparse attention and dense attention.

Page: AB-Attention summary (news.hamidun.com), "AB-Attention's three
techniques", SIP paragraph (1/pi weighting as a logit shift, "a block with a
25% probability counts as four", unbiased numerator and normaliser) and the
third paragraph (4-token blocks, original token order).  Pins: the page's
worked example against a brute-force softmax over a repeated key multiset,
all-pi=1 against dense attention, a numpy brute-force dense softmax, and a
seed-average convergence test of the HT numerator and normaliser.
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


def f64(b):
    return oracle.bf16_to_f32(b).astype(np.float64)


def _head(seed, N=64, d=16):
    rng = np.random.default_rng(seed)
    return (bits(rng.standard_normal((N, d))), bits(rng.standard_normal((N, d))),
            bits(rng.standard_normal((N, d))))


def _brute(qb, kb, vb, scale):
    q, k, v = f64(qb), f64(kb), f64(vb)
    return softmax(scale * q @ k.T, axis=1) @ v


def test_dense_matches_numpy_brute_force():
    q, k, v = _head(0, N=96, d=32)
    o = oracle.dense_attention_rows(q[:10], k, v, 0.2)
    np.testing.assert_allclose(o, _brute(q[:10], k, v, 0.2), rtol=1e-12, atol=1e-13)


def test_worked_example_quarter_probability_counts_as_four():
    """A block with pi = 0.25 weighs like its 4 tokens repeated four times."""
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        ex = json.load(f)["ht_worked_example"]
    q, k, v = _head(1, N=64, d=16)
    nkb = 16
    A = 5
    blocks = np.arange(nkb, dtype=np.int32)
    log_pi = np.zeros(nkb, np.float32)
    log_pi[A] = np.float32(math.log(ex["pi"]))
    o = oracle.sparse_attention_rows(q[:8], k, v, blocks, log_pi, 0.25)
    # brute force over the multiset: block A's tokens appear `counts_as` times
    reps = np.ones(64, int)
    reps[4 * A:4 * A + 4] = ex["counts_as"]
    kk = np.repeat(f64(k), reps, axis=0)
    vv = np.repeat(f64(v), reps, axis=0)
    ref = softmax(0.25 * f64(q[:8]) @ kk.T, axis=1) @ vv
    # the plan stores ln(0.25) in fp32: that rounding (|delta| <= 2^-24 * 1.39) moves
    # block A's weight by a relative 1e-7 at most, which bounds the difference
    bound = 2.0 ** -24 * 1.39 * 2 * np.abs(f64(v)).max()
    np.testing.assert_allclose(o, ref, rtol=0, atol=bound)
    # normaliser contribution of A is four times its dense contribution
    nhat, dhat = oracle.ht_parts(q[0], k, v, blocks, log_pi, 0.25, m_ref=0.0)
    l = 0.25 * f64(k) @ f64(q[0])
    eA = np.exp(l[4 * A:4 * A + 4]).sum()
    assert abs(dhat - (np.exp(l).sum() + 3 * eA)) <= 4 * eA * 2.0 ** -24 * 1.39 * 1.01


def test_all_pi_one_equals_dense():
    q, k, v = _head(2, N=128, d=32)
    blocks = np.arange(32, dtype=np.int32)
    o_sp = oracle.sparse_attention_rows(q[:16], k, v, blocks, np.zeros(32, np.float32), 0.17)
    o_de = oracle.dense_attention_rows(q[:16], k, v, 0.17)
    np.testing.assert_allclose(o_sp, o_de, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o_sp, _brute(q[:16], k, v, 0.17), rtol=1e-12, atol=1e-13)


def test_subset_is_softmax_over_the_selected_tokens_with_shift():
    q, k, v = _head(3, N=80, d=8)
    blocks = np.array([1, 4, 7, 19], np.int32)
    log_pi = np.array([0.0, -1.0, -0.5, -2.0], np.float32)
    o = oracle.sparse_attention_rows(q[:5], k, v, blocks, log_pi, 0.3)
    tok = np.concatenate([np.arange(4 * b, 4 * b + 4) for b in blocks])
    shift = np.repeat(log_pi.astype(np.float64), 4)
    logits = 0.3 * f64(q[:5]) @ f64(k)[tok].T - shift
    ref = softmax(logits, axis=1) @ f64(v)[tok]
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_partial_last_block_masks_missing_tokens():
    q, k, v = _head(4, N=70, d=8)   # block 17 holds tokens 68, 69 only
    blocks = np.array([0, 17], np.int32)
    o = oracle.sparse_attention_rows(q[:3], k, v, blocks, np.zeros(2, np.float32), 0.5)
    tok = np.array([0, 1, 2, 3, 68, 69])
    ref = softmax(0.5 * f64(q[:3]) @ f64(k)[tok].T, axis=1) @ f64(v)[tok]
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_empty_sample_gives_zero_output():
    q, k, v = _head(5)
    o = oracle.sparse_attention_rows(q[:4], k, v, np.zeros(0, np.int32), np.zeros(0, np.float32), 1.0)
    assert np.all(o == 0.0)


def test_ht_numerator_and_normaliser_are_unbiased_and_converge():
    """Seed means of Nhat, Dhat approach dense N, D within 4 standard errors; RMS ~ S^-1/2."""
    w = synthetic.TOY
    q, k, v = synthetic.layer_qkv_bits(w, heads=range(1))
    scores, _, _, _ = oracle.select_scores(q, k)
    qb, row_in_block = 1, 37
    s = scores[0, 0, qb]
    nkb = s.shape[0]
    n = w.budget
    p_capped, r, R, _ = oracle.pi_solve(s, n)
    qv = oracle.quantised_scores(s)
    pi = np.array([1.0 if c else r * x / R for c, x in zip(p_capped, qv)])
    kh, vh = k[0, 0], v[0, 0]
    qrow = q[0, 0, 128 * qb + row_in_block]
    scale = 1 / math.sqrt(w.d)
    # dense parts with the dense max as reference
    l = scale * f64(kh) @ f64(qrow)
    m_ref = float(l.max())
    e = np.exp(l - m_ref)
    N_dense = e @ f64(vh)
    D_dense = e.sum()
    # exact per-block contributions a_j and the Poisson-sampling standard error
    aD = e.reshape(nkb, 4).sum(1)
    aN = (e[:, None] * f64(vh)).reshape(nkb, 4, -1).sum(1)
    varD = ((1 - pi) / pi * aD ** 2).sum()
    varN = ((1 - pi)[:, None] / pi[:, None] * aN ** 2).sum(0)
    sizes = [16, 64, 256, 1024, 4096]
    rmsD = []
    accN = np.zeros_like(N_dense)
    accD = 0.0
    done = 0
    cap = nkb
    for S in sizes:
        while done < S:
            idx, lp, _, _, _ = oracle.sample_row(s, n, seed=done, row=qb, cap=cap)
            nh, dh = oracle.ht_parts(qrow, kh, vh, idx, lp, scale, m_ref)
            accN += nh
            accD += dh
            done += 1
        meanN, meanD = accN / S, accD / S
        assert abs(meanD - D_dense) <= 4 * math.sqrt(varD / S)
        assert np.all(np.abs(meanN - N_dense) <= 4 * np.sqrt(varN / S) + 1e-12)
        rmsD.append(abs(meanD - D_dense) / math.sqrt(varD))
    # independent repetitions for the rate: RMS over 32 disjoint seed batches per size
    rms = []
    for S in (16, 64, 256, 1024):
        errs = []
        for rep in range(32):
            tot = 0.0
            for t in range(S):
                idx, lp, _, _, _ = oracle.sample_row(s, n, seed=100000 + rep * 1000 + t, row=qb, cap=cap)
                tot += oracle.ht_parts(qrow, kh, vh, idx, lp, scale, m_ref)[1]
            errs.append((tot / S - D_dense) ** 2)
        rms.append(math.sqrt(np.mean(errs)))
    slope = np.polyfit(np.log([16, 64, 256, 1024]), np.log(rms), 1)[0]
    assert -0.6 <= slope <= -0.4, slope
