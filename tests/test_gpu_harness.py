"""The mass-retention harness against the oracle and against what must hold.

- Block masses from the library's dense kernel with one-hot value columns
  equal the oracle's fp64 dense attention run with the same one-hot values
  (bf16 P and bf16 output: 1e-2 relative + 1e-4 absolute), and every row
  sums to 1.
- Ideal top-k holds at least as much mass as any other selection of the same
  size (IBCS top n, block-mean top n, the systematic SIP sample), and every
  selector keeps all the mass when n covers every key block.
"""
import math

import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import harness, params_for, synthetic
from gpu_helpers import RAGGED128, SMALL128, device_bf16

pytestmark = pytest.mark.gpu

BF16_ONE = 0x3F80


def _oracle_masses(w, q, k):
    nqb, nkb = w.nqb, w.nkb
    M = np.zeros((w.B, w.H, nqb, nkb))
    scale = 1.0 / math.sqrt(w.d)
    for b in range(w.B):
        for h in range(w.H):
            for c0 in range(0, nkb, w.d):
                ncols = min(w.d, nkb - c0)
                v1 = np.zeros((w.N, w.d), np.uint16)
                t = np.arange(w.N)
                sel = (t // 4 >= c0) & (t // 4 < c0 + ncols)
                v1[t[sel], t[sel] // 4 - c0] = BF16_ONE
                o = oracle.dense_attention_rows(q[b, h], k[b, h], v1, scale)
                for qb in range(nqb):
                    rows = o[128 * qb:min(w.N, 128 * qb + 128)]
                    M[b, h, qb, c0:c0 + ncols] = rows.mean(axis=0)[:ncols]
    return M


@pytest.mark.parametrize("w", [synthetic.TOY, RAGGED128, SMALL128], ids=lambda w: w.name)
def test_block_masses_match_oracle(w):
    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w)
    M = harness.block_masses(p, device_bf16(q), device_bf16(k)).cpu().numpy()
    ref = _oracle_masses(w, q, k)
    assert np.all(np.abs(M - ref) <= 1e-2 * ref + 1e-4), float(np.abs(M - ref).max())
    assert np.allclose(ref.sum(axis=-1), 1.0, atol=1e-9)
    assert np.allclose(M.sum(axis=-1), 1.0, atol=1e-2)


@pytest.mark.parametrize("w", [synthetic.TOY, SMALL128], ids=lambda w: w.name)
def test_retention_report_invariants(w):
    q, k, v = synthetic.layer_qkv_bits(w)
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    rep, M = harness.retention_report(w, qd, kd, vd, seed=3)
    top = rep["mass_ideal_topk"]
    for key in ("mass_block_mean", "mass_ibcs_topn", "mass_sip_systematic"):
        assert rep[key] <= top + 1e-6, (key, rep[key], top)
    assert rep["mean_blocks_sip_systematic"] == w.budget
    assert 0.0 < rep["mass_ideal_topk_128token_blocks"] <= 1.0 + 1e-2
    assert abs(rep["mass_row_sum_mean"] - 1.0) < 1e-2
    # shared draws make the two samples of a query-block pair overlap more
    assert 1.0 <= rep["pair_union_over_own_paired"] < rep["pair_union_over_own_poisson"] <= 2.0
    # every key block: all selectors keep everything and reproduce dense attention
    full, _ = harness.retention_report(w, qd, kd, vd, budget=w.nkb, seed=3)
    for key in ("mass_ideal_topk", "mass_block_mean", "mass_ibcs_topn", "mass_sip_poisson",
                "mass_sip_systematic", "mass_sip_paired"):
        assert abs(full[key] - 1.0) < 1e-2, (key, full[key])
    for key in ("rel_l2_ideal_topk", "rel_l2_sip_poisson", "rel_l2_sip_systematic",
                "rel_l2_sip_paired", "rel_l2_remainder_ibcs_topn", "rel_l2_remainder_sip_poisson"):
        assert full[key] == 0.0, (key, full[key])
    assert full["pair_union_over_own_paired"] == 1.0
