"""The host-buffer step (absa_step_host) against the device-buffer calls.

Heads are independent in every stage and the draw counter uses the global
plan row, so running the step in runs of heads must give bit-for-bit the
scores, plan and output of absa_select_plan + absa_sparse_attention over the
whole problem, for every run length, with pinned or pageable host memory, and
for the paired draws too (a run starts at a head boundary, so query-block
pairs never straddle two runs).
The output is also checked against the oracle fed the GPU's plan.
"""
import numpy as np
import pytest

import oracle
from block_sparse_attention_selector_b200 import (Plan, params_for, select_plan, sparse_attention,
                                                  step_host, synthetic, workspace)
from gpu_helpers import (ATTN_MAX_ABS, ATTN_REL_L2, RAGGED128, attention_errors, device_bf16,
                         plan_to_numpy, scale_of)

pytestmark = pytest.mark.gpu

HEADS5 = synthetic.Workload("heads5_3x16x30_d128", 1, 5, 128, 3, 16, 30, 37, 3.0, 4.0, 9)


def _host(bits, pin):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t.clone()


@pytest.mark.parametrize("sampling", ["poisson", "paired"])
@pytest.mark.parametrize("w", [RAGGED128, HEADS5], ids=lambda w: w.name)
def test_step_host_equals_device_calls(w, sampling):
    import torch

    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=23, sampling=sampling)
    qd, kd, vd = device_bf16(q), device_bf16(k), device_bf16(v)
    plan_ref, s_ref, _ = select_plan(p, qd, kd)
    o_ref = sparse_attention(p, qd, kd, vd, plan_ref)
    plan_ref.check()
    ref = plan_to_numpy(plan_ref)

    bh = w.B * w.H
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    for run, pin in [(1, True), (2, True), (3, False), (bh, True), (bh + 7, True)]:
        qh, kh, vh = _host(q, pin), _host(k, pin), _host(v, pin)
        oh = torch.zeros_like(qh).pin_memory() if pin else torch.zeros_like(qh)
        qx, kx, vx = (torch.full_like(qd, float("nan")) for _ in range(3))
        ox = torch.full_like(qd, float("nan"))
        scores = torch.full_like(s_ref, -1.0)
        plan = Plan(p, qd.device)
        ws = workspace(p, qd.device)
        stream = torch.cuda.current_stream()
        step_host(p, qh, kh, vh, oh, qx, kx, vx, ox, plan, scores, ws, heads_per_run=run,
                  stream=stream, copy_in_stream=cin, copy_out_stream=cout)
        stream.synchronize()
        plan.check()
        got = plan_to_numpy(plan)
        for key in ("counts", "kv_index", "log_pi", "r_R"):
            assert np.array_equal(got[key], ref[key]), (run, key)
        assert torch.equal(scores, s_ref), run
        assert torch.equal(ox, o_ref), run
        assert torch.equal(oh, o_ref.cpu()), run

    # the output against the oracle fed the same plan
    o_or = oracle.sparse_attention(q, k, v, ref, scale_of(w))
    mx, rel = attention_errors(o_ref.float().cpu().numpy(), o_or)
    assert mx <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, (mx, rel)


def test_step_host_repeated_calls_reuse_buffers():
    """Back-to-back steps on the same device buffers: the second step's copies
    into q/k/v wait for the first step's compute, so both give the same output."""
    import torch

    w = HEADS5
    q, k, v = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=5)
    qh, kh, vh = _host(q, True), _host(k, True), _host(v, True)
    o1 = torch.zeros_like(qh).pin_memory()
    o2 = torch.zeros_like(qh).pin_memory()
    qd = torch.empty(qh.shape, dtype=torch.bfloat16, device="cuda")
    kd, vd, od = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    nqb, nkb = (w.N + 127) // 128, (w.N + 3) // 4
    scores = torch.empty((w.B, w.H, nqb, nkb), dtype=torch.float32, device="cuda")
    plan = Plan(p, "cuda")
    ws = workspace(p, "cuda")
    cin, cout = torch.cuda.Stream(), torch.cuda.Stream()
    stream = torch.cuda.current_stream()
    step_host(p, qh, kh, vh, o1, qd, kd, vd, od, plan, scores, ws, heads_per_run=2,
              stream=stream, copy_in_stream=cin, copy_out_stream=cout)
    step_host(p, qh, kh, vh, o2, qd, kd, vd, od, plan, scores, ws, heads_per_run=2,
              stream=stream, copy_in_stream=cin, copy_out_stream=cout)
    stream.synchronize()
    plan.check()
    assert torch.equal(o1, o2)
    assert bool(torch.isfinite(o1.float()).all())
