"""Pins of the oracle's SIP sampler (inclusion probabilities and draws).

Page: AB-Attention summary (news.hamidun.com), "AB-Attention's three
techniques", SIP paragraph: inclusion probability proportional to score, the
top blocks always taken, every block a nonzero chance.  Pins: the exact
integer identity sum(pi) = n, an independent fp64 bisection of
sum_j min(1, lambda q_j) = n, the published SplitMix64 outputs, and a
frequency test of the draws.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def pis(s, n):
    capped, r, R, _ = oracle.pi_solve(s, n)
    q = oracle.quantised_scores(s)
    return [1.0 if c else r * qj / R for c, qj in zip(capped, q)], capped, r, R, q


@pytest.mark.parametrize("seed,nkb,n", [(0, 128, 13), (1, 500, 40), (2, 8190, 819), (3, 64, 63),
                                        (4, 64, 1), (5, 1000, 400)])
def test_pi_sums_to_budget_exactly_and_caps_are_the_fixed_point(seed, nkb, n):
    s = synthetic.random_scores(1, nkb, seed)[0]
    capped, r, R, rounds = oracle.pi_solve(s, n)
    q = oracle.quantised_scores(s)
    # exact: |C| + r * (sum of uncapped q) / R = |C| + r = n
    assert int(capped.sum()) + r == n
    assert R == sum(qj for qj, c in zip(q, capped) if not c)
    for qj, c in zip(q, capped):
        assert (r * qj >= R) == bool(c)  # fixed point: capped <=> r q_j >= R
        if not c:
            assert 0 < r * qj < R  # 0 < pi < 1
    assert rounds >= 1


def _bisection_pi(q, n):
    """Independent characterisation: pi_j = min(1, lam q_j) with sum pi = n (fp64)."""
    q = np.asarray(q, np.float64)
    lo, hi = 0.0, n / q.min()
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if np.minimum(1.0, mid * q).sum() < n:
            lo = mid
        else:
            hi = mid
    return np.minimum(1.0, hi * q)


@pytest.mark.parametrize("seed", range(6))
def test_pi_matches_bisection_brute_force(seed):
    nkb = [16, 32, 64, 100, 128, 200][seed]
    n = [3, 5, 13, 20, 50, 199][seed]
    s = synthetic.random_scores(1, nkb, 100 + seed, concentration=2.0 + seed)[0]
    p, capped, _, _, q = pis(s, n)
    ref = _bisection_pi(q, n)
    np.testing.assert_allclose(p, ref, rtol=1e-9, atol=1e-12)


def test_pi_proportional_to_score_below_cap():
    s = np.array([0.5, 0.25, 0.125, 0.0625, 0.03125, 0.03125], np.float32)  # exact in fp32
    p, capped, r, R, q = pis(s, 2)
    # 0.5 * 2 = 1 caps block 0; the rest share r = 1 in proportion to score
    assert capped.tolist() == [True, False, False, False, False, False]
    assert r == 1 and R == 1 << 31
    assert p[1:] == [0.5, 0.25, 0.125, 0.0625, 0.0625]


def test_zero_score_keeps_a_nonzero_chance_and_unit_score_caps():
    s = np.zeros(10, np.float32)
    s[0] = 1.0
    q = oracle.quantised_scores(s)
    assert q[0] == 1 << 32 and q[1:] == [1] * 9
    p, capped, _, _, _ = pis(s, 3)
    assert capped[0] and all(0 < x < 1 for x in p[1:])
    assert abs(sum(p) - 3) < 1e-12


def test_splitmix64_published_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_reference.json")) as f:
        g = json.load(f)
    gamma = int(g["gamma"], 16)
    got = [oracle.splitmix64_mix((k * gamma) % 2**64) for k in (1, 2, 3)]
    assert got == [int(x, 16) for x in g["outputs_from_state_0"]]


def test_draws_with_seed_zero_are_the_published_splitmix64_stream():
    # mix(0) = 0, so seed 0 draws are the high halves of SplitMix64 from state 0
    with open(os.path.join(GOLDEN, "splitmix64_reference.json")) as f:
        g = json.load(f)
    for ctr, out in enumerate(g["outputs_from_state_0"]):
        assert oracle.draw_u32(0, ctr) == int(out, 16) >> 32


def test_draw_seed_selects_a_keyed_stream():
    # seed s uses the stream started from mix(s): output ctr+1 of that stream
    gamma = 0x9E3779B97F4A7C15
    for seed in (1, 17, 2**63 + 5):
        key = oracle.splitmix64_mix(seed)
        for ctr in (0, 1, 12345):
            z = oracle.splitmix64_mix((key + (ctr + 1) * gamma) % 2**64)
            assert oracle.draw_u32(seed, ctr) == z >> 32
    assert oracle.draw_u32(1, 0) != oracle.draw_u32(2, 0)


def test_sample_row_dense_short_circuit():
    s = synthetic.random_scores(1, 64, 1)[0]
    idx, lp, taken, r, R = oracle.sample_row(s, 64, seed=3, row=0, cap=64)
    assert taken == 64 and idx.tolist() == list(range(64)) and np.all(lp == 0)
    assert (r, R) == (0, 0)


def test_sample_row_structure_and_log_pi():
    nkb, n = 2000, 150
    s = synthetic.random_scores(1, nkb, 11)[0]
    p, capped, r, R, q = pis(s, n)
    cap = oracle.plan_capacity(n, nkb)
    idx, lp, taken, r2, R2 = oracle.sample_row(s, n, seed=5, row=7, cap=cap)
    assert (r2, R2) == (r, R)
    assert taken == len(idx) <= cap
    assert np.all(np.diff(idx) > 0)                    # ascending, no repeats
    assert all(capped[j] for j in np.flatnonzero(capped)) and set(np.flatnonzero(capped)) <= set(idx)
    for j, l in zip(idx, lp):
        if capped[j]:
            assert l == 0.0
        else:
            assert l < 0 and abs(float(l) - math.log(p[j])) <= 2 * np.spacing(np.float32(abs(l)))


def test_sample_row_draw_rule():
    nkb, n, seed, row = 300, 30, 9, 123
    s = synthetic.random_scores(1, nkb, 12)[0]
    _, capped, r, R, q = pis(s, n)
    idx, _, _, _, _ = oracle.sample_row(s, n, seed, row, cap=nkb)
    expect = [j for j in range(nkb)
              if capped[j] or oracle.draw_u32(seed, row * nkb + j) * R < (r * q[j]) << 32]
    assert idx.tolist() == expect


def test_inclusion_frequencies_match_pi():
    """Over 10^4 seeds each block's inclusion frequency is within 5 sigma of pi."""
    nkb, n, S = 64, 10, 10000
    s = synthetic.random_scores(1, nkb, 21)[0]
    p, _, _, _, _ = pis(s, n)
    p = np.array(p)
    hits = np.zeros(nkb)
    sizes = np.zeros(S)
    for seed in range(S):
        idx, _, taken, _, _ = oracle.sample_row(s, n, seed, 0, cap=nkb)
        hits[idx] += 1
        sizes[seed] = taken
    freq = hits / S
    sigma = np.sqrt(p * (1 - p) / S) + 1e-12
    assert np.all(np.abs(freq - p) <= 5 * sigma + 1e-12)
    var = float((p * (1 - p)).sum())
    assert abs(sizes.mean() - n) <= 5 * math.sqrt(var / S)


def test_plan_capacity_formula():
    assert oracle.plan_capacity(819, 8190) == 1088
    assert oracle.plan_capacity(13, 128) == 96
    assert oracle.plan_capacity(8190, 8190) == 8190
    assert oracle.plan_capacity(1512, 18900) == 1856   # 1512 + ceil(311.07) + 32
    assert oracle.plan_capacity(2376, 29700) == 2816   # 2376 + 390 + 32 = 2798 -> 2816


# ---------------------------------------------------------------- systematic design
# The fixed-size alternative (the SIP paragraph fixes the inclusion
# probabilities, not the design): systematic sampling with probabilities pi.
# Pins: exactly n blocks in every row, capped blocks always taken, the
# inclusion probability over the uniform U equal to pi_j (counted on a grid of
# U values), and agreement with a second formulation written with exact
# rationals (cumulative pi and the points u, u+1, ..., u+n-1).

def _systematic_by_fractions(s, n, U):
    from fractions import Fraction

    capped, r, R, _ = oracle.pi_solve(s, n)
    q = oracle.quantised_scores(s)
    u = Fraction(U, 1 << 32)
    take, cum = [], Fraction(0)
    for qj, c in zip(q, capped):
        lo = cum
        cum = cum + (1 if c else Fraction(r * qj, R))
        # points u + k, k = 0..n-1, below x: max(0, ceil(x - u)) (capped at n)
        below = lambda x: min(n, max(0, math.ceil(x - u)))
        take.append(below(cum) > below(lo))
    assert cum == n
    return np.array(take)


@pytest.mark.parametrize("seed,nkb,n", [(0, 128, 13), (1, 500, 40), (2, 8190, 819), (3, 64, 63),
                                        (4, 64, 1), (5, 1000, 400), (6, 2000, 7)])
def test_systematic_takes_exactly_n_including_every_capped_block(seed, nkb, n):
    s = synthetic.random_scores(1, nkb, seed, concentration=0.3)[0]
    capped, r, R, _ = oracle.pi_solve(s, n)
    rng = np.random.default_rng(seed)
    for U in [0, 1, (1 << 32) - 1] + rng.integers(0, 1 << 32, 5).tolist():
        take, r2, R2 = oracle.systematic_take(s, n, U)
        assert (r2, R2) == (r, R)
        assert int(take.sum()) == n
        assert bool(take[capped].all())


@pytest.mark.parametrize("seed,nkb,n", [(0, 12, 4), (1, 40, 9), (2, 16, 15), (3, 30, 1)])
def test_systematic_inclusion_probability_is_pi(seed, nkb, n):
    # over U on a grid of 4096 equally spaced values the block j is taken for
    # a set of U that is one interval or two (wrapping), of measure pi_j
    s = synthetic.random_scores(1, nkb, seed, concentration=0.5)[0]
    p, capped, r, R, q = pis(s, n)
    grid = [(i << 20) + (1 << 19) for i in range(4096)]
    counts = np.zeros(nkb)
    for U in grid:
        counts += oracle.systematic_take(s, n, U)[0]
    assert np.all(np.abs(counts - 4096 * np.array(p)) <= 2.0), (counts, p)


@pytest.mark.parametrize("seed,nkb,n", [(0, 12, 4), (1, 60, 9), (2, 33, 32), (3, 200, 17)])
def test_systematic_matches_the_rational_formulation(seed, nkb, n):
    s = synthetic.random_scores(1, nkb, seed, concentration=0.4)[0]
    rng = np.random.default_rng(100 + seed)
    for U in [0, (1 << 32) - 1] + rng.integers(0, 1 << 32, 20).tolist():
        got, _, _ = oracle.systematic_take(s, n, U)
        assert np.array_equal(got, _systematic_by_fractions(s, n, U)), U


def test_systematic_plan_row_and_layer():
    s = synthetic.random_scores(3, 300, 8, concentration=0.3)
    n, cap, seed = 20, oracle.plan_capacity(20, 300), 11
    for row in range(3):
        idx, lp, taken, r, R = oracle.sample_row(s[row], n, seed, row, cap, design="systematic")
        U = oracle.draw_u32(seed, row * 300)
        take, _, _ = oracle.systematic_take(s[row], n, U)
        assert taken == n and np.array_equal(idx, np.nonzero(take)[0])
        capped, r2, R2, _ = oracle.pi_solve(s[row], n)
        q = oracle.quantised_scores(s[row])
        for j, l in zip(idx, lp):
            want = 0.0 if capped[j] else np.float32(math.log(r * q[j] / R))
            assert l == want
    plan = oracle.sample_plan(s.reshape(1, 1, 3, 300), n, seed, cap, design="systematic")
    assert np.all(plan["counts"] == n) and plan["overflow_rows"] == 0
    idx1, _, _, _, _ = oracle.sample_row(s[1], n, seed, 1, cap, design="systematic")
    assert np.array_equal(plan["kv_index"][0, 0, 1, :n], idx1)
    # n >= nkb: every block
    idx, lp, taken, r, R = oracle.sample_row(s[0], 300, seed, 0, 300, design="systematic")
    assert taken == 300 and np.array_equal(idx, np.arange(300)) and not lp.any()


# ---------------------------------------------------------------- paired design
# Correlated draws across a pair of query blocks: blocks 2p and 2p+1 of a head
# share the uniform of every KV block, so each row is still its own Poisson
# sample with probabilities pi (the SIP paragraph's unbiasedness holds row by
# row) while the two samples nest: a block in the sample with the smaller
# pi_j is in the other.  Pins: that coupling identity on every block, the
# joint inclusion frequencies P(both) = min(pi_0, pi_1) and
# P(either) = max(pi_0, pi_1) over 10^4 seeds, and the marginals of the odd row.

def _pair_scores(nkb, seed):
    """Two correlated score rows (neighbouring query blocks attend alike)."""
    base = synthetic.random_scores(1, nkb, seed, concentration=1.5)[0].astype(np.float64)
    noise = synthetic.random_scores(1, nkb, seed + 1, concentration=1.5)[0]
    s1 = 0.7 * base + 0.3 * noise
    return np.stack([base, s1 / s1.sum()]).astype(np.float32)


def _pair_plan(s2, n, seed, design="paired"):
    nkb = s2.shape[-1]
    plan = oracle.sample_plan(s2.reshape(1, 1, 2, nkb), n, seed, nkb, design=design)
    takes = np.zeros((2, nkb), bool)
    for qb in range(2):
        takes[qb, plan["kv_index"][0, 0, qb, :plan["counts"][0, 0, qb]]] = True
    return takes, plan


def test_paired_samples_nest_block_by_block():
    nkb, n = 500, 60
    s2 = _pair_scores(nkb, 31)
    p0 = np.array(pis(s2[0], n)[0])
    p1 = np.array(pis(s2[1], n)[0])
    lo_is_0 = p0 <= p1
    for seed in range(50):
        takes, _ = _pair_plan(s2, n, seed)
        t_lo = np.where(lo_is_0, takes[0], takes[1])
        t_hi = np.where(lo_is_0, takes[1], takes[0])
        assert not np.any(t_lo & ~t_hi), seed


def test_paired_joint_inclusion_frequencies():
    nkb, n, S = 64, 10, 10000
    s2 = _pair_scores(nkb, 41)
    p0 = np.array(pis(s2[0], n)[0])
    p1 = np.array(pis(s2[1], n)[0])
    both = np.zeros(nkb)
    either = np.zeros(nkb)
    odd = np.zeros(nkb)
    union_sizes = np.zeros(S)
    for seed in range(S):
        takes, _ = _pair_plan(s2, n, seed)
        both += takes[0] & takes[1]
        either += takes[0] | takes[1]
        odd += takes[1]
        union_sizes[seed] = (takes[0] | takes[1]).sum()
    for freq, p in ((both / S, np.minimum(p0, p1)), (either / S, np.maximum(p0, p1)),
                    (odd / S, p1)):
        sigma = np.sqrt(p * (1 - p) / S) + 1e-12
        assert np.all(np.abs(freq - p) <= 5 * sigma + 1e-12)
    pm = np.maximum(p0, p1)
    assert abs(union_sizes.mean() - pm.sum()) <= 5 * math.sqrt(float((pm * (1 - pm)).sum()) / S)
    # independent draws would give sum(p0 + p1 - p0 p1) blocks in the union
    assert pm.sum() < (p0 + p1 - p0 * p1).sum() - 5 * math.sqrt(float((pm * (1 - pm)).sum()) / S)


def test_paired_rows_and_unpaired_tail():
    # even query blocks keep their own Poisson draws, odd ones take their
    # partner's counter row; with NQB odd the last block keeps its own
    nkb, n, seed, nqb = 300, 30, 5, 3
    s = synthetic.random_scores(2 * nqb, nkb, 51).reshape(1, 2, nqb, nkb)
    cap = oracle.plan_capacity(n, nkb)
    got = oracle.sample_plan(s, n, seed, cap, design="paired")
    for h in range(2):
        for qb in range(nqb):
            row = h * nqb + qb
            draw_row = row - 1 if qb % 2 == 1 else row
            idx, lp, taken, r, R = oracle.sample_row(s[0, h, qb], n, seed, draw_row, cap)
            c = got["counts"][0, h, qb]
            assert c == min(taken, cap)
            assert np.array_equal(got["kv_index"][0, h, qb, :c], idx[:c])
            assert np.array_equal(got["log_pi"][0, h, qb, :c], lp[:c])
            assert tuple(got["r_R"][0, h, qb]) == (r, R)
