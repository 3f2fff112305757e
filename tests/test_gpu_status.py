"""Device-reported errors of the selector and the bounded waits, through the C ABI.

- The wait self-test makes a bounded device wait run out on purpose: one warp
  waits on a shared-memory barrier that nothing completes, with no copy or
  MMA in flight, so the kernel gives up after the short limit, sets
  ABSA_DEVFLAG_TIMEOUT and returns; the context stays usable afterwards.
- absa_select_scores reports into the status word at the end of its
  workspace, which absa_select_check reads; each call resets it.
- absa_select_pool_kmeans followed by absa_select_block_scores computes
  exactly what absa_select_scores computes.
"""
import numpy as np
import pytest

import block_sparse_attention_selector_b200 as absa
from block_sparse_attention_selector_b200 import _abi, params_for, synthetic
from gpu_helpers import SMALL128, device_bf16

pytestmark = pytest.mark.gpu


def _stream():
    import torch

    return torch.cuda.current_stream().cuda_stream


def test_bounded_wait_runs_out_sets_the_flag_and_leaves_the_context_usable():
    import torch

    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    assert _abi.absa_selftest_wait_timeout(status.data_ptr(), 2_000_000, _stream()) == _abi.ABSA_OK
    end.record()
    torch.cuda.synchronize()
    assert int(status[0].item()) & _abi.ABSA_DEVFLAG_TIMEOUT
    # about a millisecond of clocks plus the sleep granularity of the wait loop
    assert start.elapsed_time(end) < 100.0
    # the same context still runs the library's kernels
    w = synthetic.TOY
    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w)
    scores, ws = absa.select_scores(p, device_bf16(q), device_bf16(k))
    absa.select_check(p, ws)
    s = scores.cpu().numpy()
    assert np.all(np.isfinite(s)) and np.allclose(s.sum(-1), 1.0, atol=1e-4)


def test_select_check_reads_the_workspace_status_word():
    import torch

    w = synthetic.TOY
    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w)
    qd, kd = device_bf16(q), device_bf16(k)
    scores, ws = absa.select_scores(p, qd, kd)
    assert _abi.absa_select_check(p, ws.data_ptr(), _stream()) == _abi.ABSA_OK
    # the word is the first int32 of the last 256-byte region of the workspace
    word = ws[ws.numel() - 256:ws.numel() - 252].view(torch.int32)
    word.fill_(_abi.ABSA_DEVFLAG_TIMEOUT)
    assert _abi.absa_select_check(p, ws.data_ptr(), _stream()) == _abi.ABSA_ERR_TIMEOUT
    # the next selector call resets it
    absa.select_scores(p, qd, kd, scores, ws)
    assert _abi.absa_select_check(p, ws.data_ptr(), _stream()) == _abi.ABSA_OK


@pytest.mark.parametrize("w", [synthetic.TOY, SMALL128])
def test_stage_entry_points_equal_select_scores(w):
    import torch

    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w)
    qd, kd = device_bf16(q), device_bf16(k)
    ref, _ = absa.select_scores(p, qd, kd)
    ws = absa.workspace(p)
    absa.pool_kmeans(p, qd, kd, ws)
    got = absa.block_scores(p, ws)
    absa.select_check(p, ws)
    assert torch.equal(got, ref)
