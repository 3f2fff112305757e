"""Mass-retention and error harness for the block selectors.

The AB-Attention pages compare selectors by how much of the dense attention
mass the chosen key blocks hold and by the output error against dense
attention (summary page, "AB-Attention's three techniques": ideal top-k,
block averaging, IBCS and SIP; 128- versus 4-token blocks).  This module
measures both on the GPU for one layer:

- the dense block masses M[b,h,qb,j] (mean over the valid queries of block qb
  of the softmax mass of key block j) come from the library's dense kernel
  run with one-hot value columns: with v_t = e_{j(t) - c0}, the output row of
  query i is the mass of key blocks c0 .. c0+d-1 for that query;
- the selectors at an equal number n of key blocks per query block: ideal
  top-k of M, the block-mean selector (softmax of mean query . mean key,
  top n), IBCS (the library's scores, top n), and the SIP plans of both
  sampling designs (Horvitz-Thompson weights);
- ideal top-k with 128-token key blocks at the same key fraction;
- the output error: each selection run through the library's sparse
  attention (deterministic selections with pi = 1), relative L2 against the
  library's dense output.

Selections and reductions are tensor bookkeeping on the device; every
attention and score computation runs in the library's kernels.
"""
import math

from . import (Plan, dense_reference, params_for, remainder_attention, sample_plan, select_scores,
               sparse_attention)


def block_masses(p, q, k, chunk_out=None):
    """M [B,H,NQB,NKB] fp32: dense attention mass of each key block, averaged over the valid
    queries of each query block.  Uses len(key blocks)/d dense-kernel calls."""
    import torch

    B, H, N, d = q.shape
    nqb, nkb = (N + 127) // 128, (N + 3) // 4
    dev = q.device
    M = torch.zeros((B, H, nqb, nkb), dtype=torch.float32, device=dev)
    v1 = torch.zeros_like(q)
    o = torch.empty_like(q) if chunk_out is None else chunk_out
    tok_block = torch.arange(N, device=dev) // 4
    m_valid = torch.clamp(N - 128 * torch.arange(nqb, device=dev), max=128).float()
    pad = nqb * 128 - N
    for c0 in range(0, nkb, d):
        ncols = min(d, nkb - c0)
        v1.zero_()
        sel = (tok_block >= c0) & (tok_block < c0 + ncols)
        t = torch.nonzero(sel).squeeze(1)
        v1[:, :, t, tok_block[t] - c0] = 1.0
        dense_reference(p, q, k, v1, o)
        of = o.float()
        if pad:
            of = torch.nn.functional.pad(of, (0, 0, 0, pad))
        per_qb = of.view(B, H, nqb, 128, d).sum(dim=3) / m_valid.view(1, 1, nqb, 1)
        M[..., c0:c0 + ncols] = per_qb[..., :ncols]
    return M


def plan_from_indices(p, idx):
    """A Plan holding the given ascending key-block indices [B,H,NQB,n] with pi = 1."""
    import torch

    B, H, nqb, n = idx.shape
    plan = Plan(p, idx.device, capacity=max(n, 1))
    plan.counts.fill_(n)
    plan.kv_index[..., :n] = idx.to(torch.int32)
    plan.log_pi.zero_()
    return plan


def _topn(scores, n):
    import torch

    return torch.sort(torch.topk(scores, n, dim=-1).indices, dim=-1).values


def block_mean_scores(p, q, k):
    """The block-averaging baseline: logits of the mean query of each query block against the
    mean key of each 4-token block (a softmax of these gives the same top n)."""
    import torch

    B, H, N, d = q.shape
    nqb, nkb = (N + 127) // 128, (N + 3) // 4
    qf = torch.nn.functional.pad(q.float(), (0, 0, 0, nqb * 128 - N))
    m_valid = torch.clamp(N - 128 * torch.arange(nqb, device=q.device), max=128).float()
    qbar = qf.view(B, H, nqb, 128, d).sum(dim=3) / m_valid.view(1, 1, nqb, 1)
    kf = torch.nn.functional.pad(k.float(), (0, 0, 0, nkb * 4 - N))
    kbar = kf.view(B, H, nkb, 4, d).mean(dim=3)
    return torch.matmul(qbar, kbar.transpose(-1, -2)) * p.softmax_scale


def retained_mass(M, idx, counts=None):
    """Mean over plan rows of the summed block mass of the listed blocks (entries past counts
    are ignored)."""
    import torch

    g = torch.gather(M, -1, idx.long())
    if counts is not None:
        n = idx.shape[-1]
        keep = torch.arange(n, device=idx.device).view(1, 1, 1, n) < counts.unsqueeze(-1)
        g = g * keep
    return float(g.sum(dim=-1).mean())


def rel_l2(a, b):
    a, b = a.float(), b.float()
    return float((a - b).norm() / b.norm())


def pair_union_ratio(plan, nkb):
    """Blocks in the union of the samples of query blocks 2p and 2p+1, over
    the blocks the two samples hold: what a kernel loading each pair's union
    once would compute per query block (1 when the samples coincide, 2 when
    they are disjoint)."""
    import torch

    cnt = plan.counts
    B, H, nqb = cnt.shape
    npair = nqb // 2
    if npair == 0:
        return math.nan
    taken = torch.zeros(B, H, 2 * npair, nkb + 1, dtype=torch.bool, device=cnt.device)
    cap = plan.kv_index.shape[-1]
    valid = torch.arange(cap, device=cnt.device) < cnt[..., None]
    idx = torch.where(valid, plan.kv_index.long(), nkb)[:, :, :2 * npair]
    taken.scatter_(-1, idx, True)
    taken = taken[..., :nkb].reshape(B, H, npair, 2, nkb)
    union = (taken[:, :, :, 0] | taken[:, :, :, 1]).sum()
    return float(2 * union) / float(taken.sum())


def retention_report(w, q, k, v, budget=None, seed=0):
    """One layer: retained mass and relative L2 error of every selector at n blocks."""
    import torch

    p = params_for(w, seed=seed, budget=budget)
    n = p.budget_blocks
    nkb = (w.N + 3) // 4
    M = block_masses(p, q, k)
    o_dense = dense_reference(p, q, k, v)
    out = {"workload": w.name, "heads": w.H, "budget_blocks": n, "kv_blocks": nkb,
           "key_fraction": n / nkb,
           "mass_row_sum_mean": float(M.sum(dim=-1).mean())}

    def det(name, idx):
        out[f"mass_{name}"] = retained_mass(M, idx)
        o = sparse_attention(p, q, k, v, plan_from_indices(p, idx))
        out[f"rel_l2_{name}"] = rel_l2(o, o_dense)

    det("ideal_topk", _topn(M, n))
    det("block_mean", _topn(block_mean_scores(p, q, k), n))
    scores, _ = select_scores(p, q, k)
    det("ibcs_topn", _topn(scores, n))
    # ESTRA-style remainder (the plan's blocks exact, the rest through group
    # representatives) on the IBCS top-n selection
    out["rel_l2_remainder_ibcs_topn"] = rel_l2(
        remainder_attention(p, q, k, v, plan_from_indices(p, _topn(scores, n))), o_dense)

    # 128-token key blocks at the same key fraction
    n128 = max(1, round(n / 32))
    pad = (-nkb) % 32
    M128 = torch.nn.functional.pad(M, (0, pad)).view(*M.shape[:3], -1, 32).sum(dim=-1)
    out["mass_ideal_topk_128token_blocks"] = float(torch.topk(M128, n128, dim=-1).values
                                                   .sum(dim=-1).mean())
    out["blocks_128token"] = n128

    for design in ("poisson", "systematic", "paired"):
        ps = params_for(w, seed=seed, budget=n, sampling=design)
        plan = sample_plan(ps, scores)
        plan.check()
        out[f"mass_sip_{design}"] = retained_mass(M, plan.kv_index, plan.counts)
        out[f"mean_blocks_sip_{design}"] = float(plan.counts.float().mean())
        if design != "systematic":
            out[f"pair_union_over_own_{design}"] = pair_union_ratio(plan, nkb)
        o = sparse_attention(ps, q, k, v, plan)
        out[f"rel_l2_sip_{design}"] = rel_l2(o, o_dense)
        if design == "poisson":  # the remainder estimator on the same sampled blocks
            out["rel_l2_remainder_sip_poisson"] = rel_l2(remainder_attention(ps, q, k, v, plan),
                                                         o_dense)

    top = out["mass_ideal_topk"]
    out["recall_gap_block_mean"] = top - out["mass_block_mean"]
    out["recall_gap_ibcs"] = top - out["mass_ibcs_topn"]
    out["recall_gap_ratio_ibcs_over_block_mean"] = (
        out["recall_gap_ibcs"] / out["recall_gap_block_mean"]
        if out["recall_gap_block_mean"] > 0 else math.nan)
    out["rel_l2_ratio_sip_poisson_over_topk"] = (
        out["rel_l2_sip_poisson"] / out["rel_l2_ideal_topk"]
        if out["rel_l2_ideal_topk"] > 0 else math.nan)
    return out, M
