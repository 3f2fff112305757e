"""The allocation-free selector entry point (absa_select_scores_static).

It exists for callers that cannot obtain extra device memory (a plugin host
that only hands over its input and output tensors, or code running under a
memory manager it cannot call): the workspace comes from an array compiled
into the library.  This file checks, through the C ABI, that it returns
exactly what absa_select_scores returns (both run the same kernels, which use
no atomics, on the same inputs, so the scores are bit-identical), on several
calls in a row that share that array, that the array's status word reads
clean afterwards, and that a problem needing more scratch than the array
holds is refused up front.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

from block_sparse_attention_selector_b200 import _abi, params_for, synthetic
from gpu_helpers import SMALL128, device_bf16

pytestmark = pytest.mark.gpu


def _scores_both_ways(w, seed=0):
    import torch

    q, k, _ = synthetic.layer_qkv_bits(w)
    p = params_for(w, seed=seed)
    qd, kd = device_bf16(q), device_bf16(k)
    shape = (w.B, w.H, w.nqb, w.nkb)
    ref = torch.empty(shape, dtype=torch.float32, device="cuda")
    got = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
    ws_bytes = _abi.absa_workspace_bytes(p)
    assert 0 < ws_bytes <= _abi.ABSA_STATIC_SCRATCH_BYTES
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert _abi.absa_select_scores(p, qd.data_ptr(), kd.data_ptr(), ref.data_ptr(), ws.data_ptr(),
                                   ws_bytes, stream) == _abi.ABSA_OK
    assert _abi.absa_select_scores_static(p, qd.data_ptr(), kd.data_ptr(), got.data_ptr(),
                                          stream) == _abi.ABSA_OK
    # the status word inside the built-in array (no bounded wait gave up)
    assert _abi.absa_select_check(p, None, stream) == _abi.ABSA_OK
    torch.cuda.synchronize()
    return got.cpu().numpy(), ref.cpu().numpy()


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    # consecutive calls share the built-in array: a larger problem, a smaller
    # one, then the larger one again must each match the regular entry point
    for w in (SMALL128, synthetic.TOY, SMALL128):
        got, ref = _scores_both_ways(w)
        assert np.all(np.isfinite(got))
        assert np.array_equal(got, ref)


def test_static_scratch_refuses_problems_larger_than_the_array():
    w = synthetic.WAN480  # needs far more than 64 MiB of workspace
    p = params_for(w)
    assert _abi.absa_workspace_bytes(p) > _abi.ABSA_STATIC_SCRATCH_BYTES
    assert _abi.absa_select_scores_static(p, 16, 16, 16, None) == _abi.ABSA_ERR_WORKSPACE
