"""Host logic of the mass-retention harness (no GPU): the query-block pair
union ratio that the harness reports for the Poisson and paired SIP designs.

For query blocks 2p and 2p+1 of a head with samples S0 and S1 it is
sum |S0 u S1| * 2 / sum (|S0| + |S1|): 1 when every pair's samples coincide,
2 when they are disjoint.  A last unpaired query block (odd NQB) is left out,
and entries past a row's count are ignored.
"""
import types

import pytest
import torch

from block_sparse_attention_selector_b200.harness import pair_union_ratio


def _plan(rows, cap, nkb_pad=0):
    """rows: [B][H][NQB] lists of block ids -> object with counts and kv_index."""
    B, H, nqb = len(rows), len(rows[0]), len(rows[0][0])
    counts = torch.zeros(B, H, nqb, dtype=torch.int32)
    kv = torch.full((B, H, nqb, cap), nkb_pad, dtype=torch.int32)
    for b in range(B):
        for h in range(H):
            for q in range(nqb):
                ids = rows[b][h][q]
                counts[b, h, q] = len(ids)
                kv[b, h, q, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
    return types.SimpleNamespace(counts=counts, kv_index=kv)


def test_identical_and_disjoint_pairs():
    same = _plan([[[[1, 4, 7], [1, 4, 7]]]], cap=4)
    assert pair_union_ratio(same, 8) == 1.0
    disjoint = _plan([[[[0, 1], [2, 3]]]], cap=4)
    assert pair_union_ratio(disjoint, 8) == 2.0


def test_partial_overlap_odd_tail_and_stale_entries():
    # pair (0,1): union {0,1,2,3}, own 3 + 3; the fifth query block has no
    # partner and is left out; entries past the counts (filled with 5) ignored
    plan = _plan([[[[0, 1, 2], [1, 2, 3], [6], [6], [0, 1, 2, 3, 4]]]], cap=6, nkb_pad=5)
    assert pair_union_ratio(plan, 8) == pytest.approx((4 + 1) * 2 / (6 + 2))


def test_pairs_stay_within_a_head():
    # two heads of two query blocks each: pairs never mix heads
    plan = _plan([[[[0], [0]], [[1], [2]]]], cap=2)
    assert pair_union_ratio(plan, 4) == pytest.approx((1 + 2) * 2 / 4)


def test_single_query_block_has_no_pair():
    import math

    assert math.isnan(pair_union_ratio(_plan([[[[0, 1]]]], cap=2), 4))
