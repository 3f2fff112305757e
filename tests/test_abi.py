"""The C-ABI library loads, exports every entry point include/absa.h declares,
and rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

import oracle
from block_sparse_attention_selector_b200 import _abi, build, make_params, synthetic

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def header_functions():
    with open(os.path.join(ROOT, "include", "absa.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(absa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = header_functions()
    assert set(names) == set(_abi.EXPORTED)
    for name in names:
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    assert "sm_100a" in _abi.version()
    for code in range(8):
        assert _abi.status_string(code).startswith("ABSA_")


def _p(w=synthetic.WAN480, **kw):
    p = make_params(w.B, w.H, w.N, w.d, w.T, w.Hg, w.Wg, w.budget)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("w", [synthetic.TOY, synthetic.WAN480, synthetic.WAN720, synthetic.HUNYUAN720])
def test_plan_capacity_matches_oracle_rule(L, w):
    p = _p(w)
    assert _abi.absa_check_params(p) == _abi.ABSA_OK
    assert _abi.absa_plan_capacity(p) == oracle.plan_capacity(w.budget, w.nkb)
    for n in (1, 2, 82, 164, 410, 2048, w.nkb - 1, w.nkb, w.nkb + 5):
        p.budget_blocks = n
        assert _abi.absa_plan_capacity(p) == oracle.plan_capacity(n, w.nkb)


def test_workspace_bytes_covers_layout(L):
    w = synthetic.WAN480
    p = _p(w)
    BH = w.B * w.H
    nkr = (w.nkb + 255) // 256
    need = (2 * BH * w.nkb * w.d * 2 + BH * w.nqb * 8 * w.d * (4 + 2 + 2) + BH * w.nqb * 8 * 4
            + BH * w.nqb * 128 + 2 * BH * nkr * w.nqb * 8 * 4 + BH * w.nqb * 8 * 4 + 4)
    got = _abi.absa_workspace_bytes(p)
    assert need <= got <= need + 11 * 256


@pytest.mark.parametrize("w", [synthetic.TOY, synthetic.WAN480, synthetic.HUNYUAN720],
                         ids=lambda w: w.name)
def test_remainder_workspace_bytes_match_the_documented_layout(L, w):
    """mu, nu (bf16 [B,H,G,d]), var and count ([B,H,G], 4 bytes each), every region at a
    256-byte boundary, G = ceil(NKB / 32)."""
    G = (w.nkb + 31) // 32
    n = w.B * w.H * G
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert _abi.absa_remainder_workspace_bytes(_p(w)) == 2 * up(n * w.d * 2) + 2 * up(n * 4)


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, _abi.ABSA_ERR_UNSUPPORTED),
    ("q_block", 64, _abi.ABSA_ERR_UNSUPPORTED),
    ("kv_block", 8, _abi.ABSA_ERR_UNSUPPORTED),
    ("n_clusters", 4, _abi.ABSA_ERR_UNSUPPORTED),
    ("N", 0, _abi.ABSA_ERR_INVALID_ARG),
    ("T", 20, _abi.ABSA_ERR_INVALID_ARG),          # grid no longer multiplies to N
    ("budget_blocks", 0, _abi.ABSA_ERR_INVALID_ARG),
    ("kmeans_iters", 0, _abi.ABSA_ERR_INVALID_ARG),
    ("softmax_scale", float("nan"), _abi.ABSA_ERR_INVALID_ARG),
    ("sampling", 3, _abi.ABSA_ERR_INVALID_ARG),
    ("sampling", -1, _abi.ABSA_ERR_INVALID_ARG),
])
def test_bad_params_rejected(L, field, value, code):
    p = _p(**{field: value})
    assert _abi.absa_check_params(p) == code
    assert _abi.absa_plan_capacity(p) == -1
    assert _abi.absa_workspace_bytes(p) == 0


def test_too_many_kv_blocks_unsupported(L):
    p = make_params(1, 1, 4 * 49153, 128, 1, 1, 4 * 49153, 10)
    assert _abi.absa_check_params(p) == _abi.ABSA_ERR_UNSUPPORTED


def test_entry_points_reject_null_and_misaligned_pointers_before_cuda(L):
    p = _p(synthetic.TOY)
    plan = _abi.absa_plan(4, 128, 96, None, None, None, None, None)
    assert _abi.absa_select_scores(p, None, None, None, None, 0, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_sample_plan(p, 16, plan, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_sparse_attention(p, 16, 16, 16, plan, 16, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_dense_reference(p, 16, 16, 8, 16, None, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_dense_reference(p, None, 16, 16, 16, None, None) == _abi.ABSA_ERR_INVALID_ARG
    ws = _abi.absa_workspace_bytes(p)
    assert _abi.absa_select_scores(p, 16, 16, 16, 16, ws - 1, None) == _abi.ABSA_ERR_WORKSPACE
    # a plan whose shape does not match the parameters
    bad = _abi.absa_plan(5, 128, 96, 16, 16, 16, 16, 16)
    assert _abi.absa_sparse_attention(p, 16, 16, 16, bad, 16, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_plan_check(_abi.absa_plan(), None) == _abi.ABSA_ERR_INVALID_ARG
    # the pair-union attention: same checks, and a capacity above its union list
    pairs = _abi.absa_sparse_attention_pairs
    assert pairs(p, 16, 16, 16, plan, 16, None) == _abi.ABSA_ERR_INVALID_ARG
    assert pairs(p, 16, 16, 16, bad, 16, None) == _abi.ABSA_ERR_INVALID_ARG
    assert pairs(p, 16, 16, 8, _abi.absa_plan(4, 128, 96, 16, 16, 16, 16, 16), 16,
                 None) == _abi.ABSA_ERR_INVALID_ARG
    wide = _abi.absa_plan(4, 128, 3073, 16, 16, 16, 16, 16)
    assert pairs(p, 16, 16, 16, wide, 16, None) == _abi.ABSA_ERR_UNSUPPORTED
    # the remainder attention: workspace size, null and short workspaces
    rb = _abi.absa_remainder_workspace_bytes(p)
    assert rb > 0 and _abi.absa_remainder_workspace_bytes(_p(N=0)) == 0
    rem = _abi.absa_remainder_attention
    ok_plan = _abi.absa_plan(4, 128, 96, 16, 16, 16, 16, 16)
    assert rem(p, 16, 16, 16, ok_plan, 16, None, rb, None) == _abi.ABSA_ERR_INVALID_ARG
    assert rem(p, 16, 16, 16, ok_plan, 16, 16, rb - 1, None) == _abi.ABSA_ERR_WORKSPACE
    assert rem(p, 16, 16, 16, bad, 16, 16, rb, None) == _abi.ABSA_ERR_INVALID_ARG
    # the host-buffer step: null host pointers, an empty head run, a short workspace
    good = _abi.absa_plan(4, 128, 96, 16, 16, 16, 16, 16)
    step = _abi.absa_step_host
    assert step(p, None, 16, 16, 16, 16, 16, 16, 16, 16, good, 16, ws, 4, None, None,
                None) == _abi.ABSA_ERR_INVALID_ARG
    assert step(p, 16, 16, 16, 16, 16, 16, 8, 16, 16, good, 16, ws, 4, None, None,
                None) == _abi.ABSA_ERR_INVALID_ARG
    assert step(p, 16, 16, 16, 16, 16, 16, 16, 16, 16, good, 16, ws, 0, None, None,
                None) == _abi.ABSA_ERR_INVALID_ARG
    assert step(p, 16, 16, 16, 16, 16, 16, 16, 16, 16, good, 16, ws - 1, 4, None, None,
                None) == _abi.ABSA_ERR_WORKSPACE
    assert step(p, 16, 16, 16, 16, 16, 16, 16, 16, 16, bad, 16, ws, 4, None, None,
                None) == _abi.ABSA_ERR_INVALID_ARG
    # the two selector stages, the selector check and the wait self-test
    assert _abi.absa_select_pool_kmeans(p, None, 16, 16, ws, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_select_pool_kmeans(p, 16, 16, 8, ws, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_select_pool_kmeans(p, 16, 16, 16, ws - 1, None) == _abi.ABSA_ERR_WORKSPACE
    assert _abi.absa_select_block_scores(p, None, 16, ws, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_select_block_scores(p, 16, 16, ws - 1, None) == _abi.ABSA_ERR_WORKSPACE
    assert _abi.absa_select_check(p, 8, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_select_check(_p(synthetic.WAN480), None, None) == _abi.ABSA_ERR_WORKSPACE
    assert _abi.absa_selftest_wait_timeout(None, 1000, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_selftest_wait_timeout(16, 0, None) == _abi.ABSA_ERR_INVALID_ARG
    assert _abi.absa_selftest_wait_timeout(16, 2_000_000_001, None) == _abi.ABSA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "libabsa.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(ImportError):
        _abi.lib()


def test_params_struct_matches_the_header(L):
    # the Python mirror of absa_params has the C layout: 12 int32, u64 seed, float scale,
    # int32 sampling (64 bytes); every sampling design validates
    assert ctypes.sizeof(_abi.absa_params) == 64
    assert _abi.absa_params.sampling.offset == 60
    for design in ("poisson", "systematic", "paired"):
        p = make_params(1, 2, 512, 64, 4, 8, 16, 13, sampling=design)
        assert _abi.absa_check_params(p) == _abi.ABSA_OK
