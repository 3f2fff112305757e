"""GPU pair-union sparse attention (absa_sparse_attention_pairs) against the oracle.

The pair-union form runs one CTA per pair of query blocks (2p, 2p+1) of a
head over the union of the two plan rows; a block that one row lacks gets
the logit bias -inf in that row's softmax.  Each row's output must still be
the HT attention over its own entries: within max-abs 1e-2 and relative L2
5e-3 of the oracle's fp64 output, whatever the two rows hold (empty,
identical, nested, disjoint, unsorted, repeated, out of range), and the
single-block kernel (absa_sparse_attention) must meet the same bar on the
same plans.
"""
import dataclasses
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (AbsaError, _abi, params_for, select_plan,
                                                  sparse_attention, sparse_attention_pairs,
                                                  synthetic)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, RAGGED64, RAGGED128, SMALL128,
                         attention_errors, device_bf16, gpu_out_f64, load_case, plan_from_oracle)

pytestmark = pytest.mark.gpu

CASES = [synthetic.TOY, RAGGED64, RAGGED128, SMALL128]


def _assert_close(o_gpu, o_ref, what):
    mx, rel = attention_errors(o_gpu, o_ref)
    assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, f"{what}: max-abs {mx:.3g}, rel-L2 {rel:.3g}"


def _run(p, q, k, v, ref, pairs=True):
    plan = plan_from_oracle(p, ref)
    fn = sparse_attention_pairs if pairs else sparse_attention
    o = fn(p, device_bf16(q), device_bf16(k), device_bf16(v), plan)
    return plan, gpu_out_f64(o)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_paired_plan_matches_oracle(w):
    """An oracle plan drawn with the paired design (odd NQB in RAGGED64 and
    RAGGED128: the last query block has no partner)."""
    q, k, v, _ = load_case(w)
    s_ref, _, _, _ = oracle.select_scores(q, k)
    cap = oracle.plan_capacity(w.budget, w.nkb)
    ref = oracle.sample_plan(s_ref, w.budget, 3, cap, design="paired")
    p = params_for(w, seed=3, sampling="paired")
    plan, o = _run(p, q, k, v, ref)
    plan.check()
    o_ref = oracle.sparse_attention(q, k, v, ref)
    _assert_close(o, o_ref, w.name)
    # the single-block kernel on the same plan agrees too
    _, o1 = _run(p, q, k, v, ref, pairs=False)
    _assert_close(o1, o_ref, w.name + " single")


def _pair_rows(rng, kind, nkb, cap):
    """Two plan rows (ids, ln pi) for one query-block pair."""
    def pick(c, pool=None):
        pool = np.arange(nkb) if pool is None else pool
        return np.sort(rng.choice(pool, c, replace=False)).astype(np.int32)

    if kind == "empty_both":
        a, b = pick(0), pick(0)
    elif kind == "empty_a":
        a, b = pick(0), pick(33)
    elif kind == "empty_b":
        a, b = pick(47), pick(0)
    elif kind == "same_single":
        a = pick(1)
        b = a.copy()
    elif kind == "identical":
        a = pick(min(65, cap))
        b = a.copy()
    elif kind == "nested":
        a = pick(cap)
        b = np.sort(rng.choice(a, 40, replace=False)).astype(np.int32)
    elif kind == "disjoint_full":
        perm = rng.permutation(nkb)
        a, b = np.sort(perm[:cap]).astype(np.int32), np.sort(perm[cap:2 * cap]).astype(np.int32)
    elif kind == "overlap":
        a = pick(min(80, cap))
        b = np.union1d(rng.choice(a, 50, replace=False), pick(20)).astype(np.int32)[:cap]
    elif kind == "unsorted":
        a = pick(20)[::-1].copy()
        b = pick(30)
    elif kind == "repeated":
        a = pick(17)
        b = np.array([5, 5, 7, 7, 7, 9], np.int32)
    else:
        raise ValueError(kind)
    la = np.log(rng.uniform(0.05, 1.0, len(a))).astype(np.float32)
    lb = np.log(rng.uniform(0.05, 1.0, len(b))).astype(np.float32)
    if len(a):
        la[0] = np.float32(math.log(0.25))
    if kind in ("identical", "same_single"):
        lb = la.copy()
    return a, la, b, lb


KINDS = ["empty_both", "empty_a", "empty_b", "same_single", "identical", "nested",
         "disjoint_full", "overlap", "unsorted", "repeated"]


def _hand_plan(w, cap, seed, kinds):
    B, H, nqb = w.B, w.H, w.nqb
    counts = np.zeros((B, H, nqb), np.int32)
    idx = np.zeros((B, H, nqb, cap), np.int32)
    lp = np.zeros((B, H, nqb, cap), np.float32)
    rng = np.random.default_rng(seed)
    i = 0
    for b in range(B):
        for h in range(H):
            for qb in range(0, nqb, 2):
                a, la, bb, lb = _pair_rows(rng, kinds[i % len(kinds)], w.nkb, cap)
                i += 1
                counts[b, h, qb] = len(a)
                idx[b, h, qb, :len(a)] = a
                lp[b, h, qb, :len(a)] = la
                if qb + 1 < nqb:
                    counts[b, h, qb + 1] = len(bb)
                    idx[b, h, qb + 1, :len(bb)] = bb
                    lp[b, h, qb + 1, :len(bb)] = lb
    return dict(counts=counts, kv_index=idx, log_pi=lp, r_R=np.zeros((B, H, nqb, 2), np.uint64))


@pytest.mark.parametrize("shift", range(len(KINDS)))
def test_pairs_of_every_kind(shift):
    """Hand-made pairs on a 16-query-block head layout: every kind of pair at
    every pair position (the kinds rotate with `shift`), full-capacity rows
    whose union is twice the capacity, rows out of order and repeated ids."""
    w = SMALL128
    q, k, v, _ = load_case(w)
    cap = 96
    kinds = KINDS[shift:] + KINDS[:shift]
    ref = _hand_plan(w, cap, 10 + shift, kinds)
    p = params_for(w, sampling="paired")
    plan, o = _run(p, q, k, v, ref)
    plan.check()
    o_ref = oracle.sparse_attention(q, k, v, ref)
    _assert_close(o, o_ref, f"kinds from {kinds[0]}")
    _, o1 = _run(p, q, k, v, ref, pairs=False)
    _assert_close(o1, o_ref, f"single-block kernel, kinds from {kinds[0]}")
    counts = ref["counts"]
    for h in range(w.H):
        for qb in range(w.nqb):
            if counts[0, h, qb] == 0:
                assert np.all(o[0, h, 128 * qb:128 * qb + 128] == 0), (h, qb)


def test_pairs_odd_layout_with_partial_key_block():
    """RAGGED64: 3 query blocks per head (the last has no partner and 17 valid
    rows) and 69 key blocks, the last holding one token."""
    w = RAGGED64
    q, k, v, _ = load_case(w)
    cap = 40
    rng = np.random.default_rng(4)
    B, H, nqb = w.B, w.H, w.nqb
    counts = np.zeros((B, H, nqb), np.int32)
    idx = np.zeros((B, H, nqb, cap), np.int32)
    lp = np.zeros((B, H, nqb, cap), np.float32)
    for h in range(H):
        for qb in range(nqb):
            c = [cap, 25, 33][(h + qb) % 3]
            ids = np.union1d(rng.choice(w.nkb - 1, c - 1, replace=False), [w.nkb - 1])
            counts[0, h, qb] = len(ids)
            idx[0, h, qb, :len(ids)] = ids
            lp[0, h, qb, :len(ids)] = np.log(rng.uniform(0.1, 1.0, len(ids)))
    ref = dict(counts=counts, kv_index=idx, log_pi=lp, r_R=np.zeros((B, H, nqb, 2), np.uint64))
    plan, o = _run(params_for(w, sampling="paired"), q, k, v, ref)
    plan.check()
    _assert_close(o, oracle.sparse_attention(q, k, v, ref), w.name)


def test_paired_bad_rows_zero_only_themselves():
    """A count above capacity in one row and an index out of range in another
    reject those rows only: their partners keep their own attention."""
    w = SMALL128
    q, k, v, _ = load_case(w)
    cap = 64
    ref = _hand_plan(w, cap, 3, ["overlap", "nested", "identical"])
    bad = {k2: v2.copy() for k2, v2 in ref.items()}
    bad["counts"][0, 0, 1] = cap + 1              # row B of pair 0 of head 0
    bad["kv_index"][0, 1, 4, 0] = -3              # row A of pair 2 of head 1
    bad["kv_index"][0, 1, 7, 1] = w.nkb           # row B of pair 3 of head 1
    p = params_for(w, sampling="paired")
    plan, o = _run(p, q, k, v, bad)
    with pytest.raises(AbsaError) as e:
        plan.check()
    assert e.value.code == _abi.ABSA_ERR_BAD_PLAN
    for h, qb in ((0, 1), (1, 4), (1, 7)):
        assert np.all(o[0, h, 128 * qb:128 * qb + 128] == 0), (h, qb)
    o_ref = oracle.sparse_attention(q, k, v, ref)
    for h, qb in ((0, 0), (1, 5), (1, 6), (0, 2), (1, 15)):
        rows = slice(128 * qb, 128 * qb + 128)
        _assert_close(o[:, h, rows], o_ref[:, h, rows], f"partner row {h},{qb}")


def test_capacity_beyond_union_limit_is_unsupported():
    """A plan with capacity 3100 (twice that exceeds the union list the pair
    kernel keeps in shared memory) is refused before any launch; the
    single-block kernel runs it."""
    w = SMALL128
    q, k, v, _ = load_case(w)
    ref = _hand_plan(w, 96, 5, KINDS)
    cap = 3100
    for key in ("kv_index", "log_pi"):
        a = ref[key]
        wide = np.zeros(a.shape[:3] + (cap,), a.dtype)
        wide[..., :a.shape[-1]] = a
        ref[key] = wide
    p = params_for(w, sampling="paired")
    with pytest.raises(AbsaError) as e:
        _run(p, q, k, v, ref)
    assert e.value.code == _abi.ABSA_ERR_UNSUPPORTED
    plan, o = _run(p, q, k, v, ref, pairs=False)
    plan.check()
    _assert_close(o, oracle.sparse_attention(q, k, v, ref), "capacity 3100")


def test_hunyuan720_paired_layer_sampled_rows():
    """The HunyuanVideo 720p layer (929 query blocks per head: the last one has
    no partner and 16 valid rows) through select_plan and sparse_attention
    with the paired design; the oracle recomputes the attention of both rows
    of the first, a middle and the last pair of heads 0 and 23 from the
    GPU's plan."""
    import torch

    w = synthetic.HUNYUAN720
    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=w.seed, sampling="paired")
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan, _, _ = select_plan(p, qd, kd)
    o = sparse_attention_pairs(p, qd, kd, vd, plan)
    torch.cuda.synchronize()
    plan.check()
    counts = plan.counts.cpu().numpy()
    scale = 1.0 / math.sqrt(w.d)
    for h in (0, w.H - 1):
        for qb in (0, 1, 464, 465, w.nqb - 1):
            c = int(counts[0, h, qb])
            idx = plan.kv_index[0, h, qb, :c].cpu().numpy()
            lp = plan.log_pi[0, h, qb, :c].cpu().numpy()
            m = min(128, w.N - 128 * qb)
            rows = slice(128 * qb, 128 * qb + m)
            o_ref = oracle.sparse_attention_rows(q[0, h, rows], k[0, h], v[0, h], idx, lp, scale)
            mx, rel = attention_errors(o[0, h, rows].float().cpu().numpy(), o_ref)
            assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (h, qb, mx, rel)


def test_wan480_paired_matches_independent_kernel_on_same_plan():
    """Wan2.1 480p cut to 8 heads: the pair kernel and the single-block kernel
    on one paired plan agree within the attention bar everywhere (they differ
    only in the order of the sums and the lazy-max points)."""
    import torch

    w = dataclasses.replace(synthetic.WAN480, H=8)
    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=5, sampling="paired")
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan, _, _ = select_plan(p, qd, kd)
    o2 = sparse_attention_pairs(p, qd, kd, vd, plan)
    o1 = sparse_attention(p, qd, kd, vd, plan)
    torch.cuda.synchronize()
    plan.check()
    d = (o2.float() - o1.float()).abs()
    assert float(d.max()) <= ATTN_MAX_ABS
    rel = float(torch.linalg.vector_norm(d) / torch.linalg.vector_norm(o1.float()))
    assert rel <= ATTN_REL_L2, rel
