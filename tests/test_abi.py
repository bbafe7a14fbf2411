"""The C ABI without a GPU: the library loads, exports every declared entry point, and rejects
bad arguments on the host before any launch."""
import json
import os

import pytest

import exact_io_aware_43_b200 as fa

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
A = 1 << 20  # a 16-byte aligned fake device address (never dereferenced: checks run first)


def test_exports_every_declared_symbol():
    names = fa.header_functions()
    assert {"fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_last_error"} <= set(names)
    L = fa.lib()
    for n in names:
        assert hasattr(L, n), n


def test_starve_test_build_exports_the_same_symbols():
    """The test-only build used by the bounded-wait test loads and exports the same entry points
    (it differs from the product library by one left-out copy in the forward)."""
    import ctypes

    from exact_io_aware_43_b200.build import STARVE_PATH
    L = ctypes.CDLL(STARVE_PATH)
    for n in fa.header_functions():
        assert hasattr(L, n), n


def test_version():
    assert fa.fa_version() >= 100


def test_workspace_size_formula():
    B, H, N, d = 2, 16, 8192, 128
    npad = (N + 127) // 128 * 128
    # fp32 dQ accumulator + two fp32 row vectors; d = 64 and 128 add the row statistics as 32
    # bytes of MMA operand per padded row
    want = B * H * N * d * 4 + 2 * B * H * npad * 4 + B * H * npad * 32
    assert fa.fa_bwd_workspace_size(B, H, N, d) == want
    assert fa.fa_bwd_workspace_size(B, H, N, 64) == B * H * N * 64 * 4 + 2 * B * H * npad * 4 + \
        B * H * npad * 32
    assert fa.fa_bwd_workspace_size(B, H, N, 256) == B * H * N * 256 * 4 + 2 * B * H * npad * 4
    # ragged N: the row vectors are padded to 128
    got = fa.fa_bwd_workspace_size(1, 1, 129, 64)
    assert got >= 129 * 64 * 4 + 2 * 256 * 4
    for bad in ((0, 1, 1, 64), (1, 0, 1, 64), (1, 1, 0, 64), (1, 1, 8, 96)):
        assert fa.fa_bwd_workspace_size(*bad) == 0


def test_workspace_is_linear_not_quadratic():
    """The naive score matrix at B*H = 32, N = 8192 would take about 4 GB (the pages' example);
    the backward's whole workspace is O(N) per head and a small fraction of it."""
    g = json.load(open(os.path.join(GOLDEN, "naive_score_matrix_bytes.json")))
    ws = fa.fa_bwd_workspace_size(2, 16, 8192, 128)
    assert ws * 20 < g["bytes"]
    # doubling N doubles (not quadruples) the workspace
    assert fa.fa_bwd_workspace_size(2, 16, 16384, 128) == 2 * ws


def fwd(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, causal=0, scale=0.125, stream=None)
    a.update(kw)
    return fa.fa_fwd(**a)


def fwd_fp8(**kw):
    a = dict(q8=A, k8=A, v8=A, q_scale=0.01, k_scale=0.01, v_scale=0.01, o=A, lse=A, B=1, H=1,
             N=128, d=64, causal=0, scale=0.125, stream=None)
    a.update(kw)
    return fa.fa_fwd_fp8(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(q8=None), fa.FA_ERR_INVALID_ARG),
    (dict(v8=None), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(q_scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(k_scale=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(v_scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(k8=A + 1), fa.FA_ERR_MISALIGNED),
    (dict(lse=A + 4), fa.FA_ERR_MISALIGNED),
])
def test_fwd_fp8_rejects(kw, code):
    assert fwd_fp8(**kw) == code
    assert fa.fa_last_error() != ""


def test_partial_and_merge_reject_bad_arguments():
    P = dict(q=A, k=A, v=A, o_part=A, lse_part=A, B=1, H=2, H_kv=1, Nq=64, Nk=128, d=128,
             causal=1, scale=0.1, stream=None)
    assert fa.fa_fwd_partial(**{**P, "o_part": None}) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_partial(**{**P, "Nq": 200}) == fa.FA_ERR_INVALID_ARG  # causal, Nq > Nk
    assert fa.fa_fwd_partial(**{**P, "H_kv": 3}) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_partial(**{**P, "d": 96}) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_partial(**{**P, "lse_part": A + 4}) == fa.FA_ERR_MISALIGNED
    M = dict(o_parts=A, lse_parts=A, n_parts=2, o=A, lse=A, rows=100, d=64, stream=None)
    assert fa.fa_merge_partials(**{**M, "n_parts": 0}) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_merge_partials(**{**M, "rows": 0}) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_merge_partials(**{**M, "d": 32}) == fa.FA_ERR_UNSUPPORTED
    assert fa.fa_merge_partials(**{**M, "o": None}) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_merge_partials(**{**M, "o": A + 2}) == fa.FA_ERR_MISALIGNED


def test_selftest_exp2_rejects_bad_arguments():
    assert fa.fa_selftest_exp2_fma(None, A, 4, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_selftest_exp2_fma(A, A, -1, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_selftest_exp2_fma(A, A, 0, None) == fa.FA_OK  # nothing to do, nothing launched


def bwd(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, H=1, N=128, d=64, causal=0,
             scale=0.125, workspace=A, workspace_bytes=1 << 30, stream=None)
    a.update(kw)
    return fa.fa_bwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(lse=None), fa.FA_ERR_INVALID_ARG),
    (dict(B=0), fa.FA_ERR_INVALID_ARG),
    (dict(N=0), fa.FA_ERR_INVALID_ARG),
    (dict(N=-5), fa.FA_ERR_INVALID_ARG),
    (dict(d=96), fa.FA_ERR_UNSUPPORTED),
    (dict(d=32), fa.FA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(q=A + 8), fa.FA_ERR_MISALIGNED),
    (dict(o=A + 2), fa.FA_ERR_MISALIGNED),
])
def test_fwd_rejects(kw, code):
    assert fwd(**kw) == code
    assert fa.fa_last_error() != ""


@pytest.mark.parametrize("kw,code", [
    (dict(dO=None), fa.FA_ERR_INVALID_ARG),
    (dict(dq=None), fa.FA_ERR_INVALID_ARG),
    (dict(d=100), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=A + 4), fa.FA_ERR_MISALIGNED),
    (dict(workspace=None), fa.FA_ERR_WORKSPACE),
    (dict(workspace=A + 8), fa.FA_ERR_WORKSPACE),
    (dict(workspace_bytes=100), fa.FA_ERR_WORKSPACE),
])
def test_bwd_rejects(kw, code):
    assert bwd(**kw) == code
    assert fa.fa_last_error() != ""


def test_timer_read_rejects_bad_kind():
    import ctypes
    n, ms = ctypes.c_int(0), ctypes.c_double(0)
    assert fa.lib().fa_timer_read(7, ctypes.byref(n), ctypes.byref(ms)) == fa.FA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "LIB_PATH", "/nonexistent/libfattn.so")
    with pytest.raises(fa.FattnError):
        fa.lib()


def fwd_gqa(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=4, H_kv=2, N=128, d=64, causal=0, scale=0.125,
             stream=None)
    a.update(kw)
    return fa.fa_fwd_gqa(**a)


def bwd_gqa(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, dO=A, dq=A, dk=A, dv=A, B=1, H=4, H_kv=2, N=128, d=64,
             causal=0, scale=0.125, workspace=A, workspace_bytes=1 << 30, stream=None)
    a.update(kw)
    return fa.fa_bwd_gqa(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(H_kv=3), fa.FA_ERR_INVALID_ARG),     # does not divide H
    (dict(H_kv=0), fa.FA_ERR_INVALID_ARG),
    (dict(H_kv=-2), fa.FA_ERR_INVALID_ARG),
    (dict(H_kv=8), fa.FA_ERR_INVALID_ARG),     # more key/value heads than query heads
    (dict(k=None), fa.FA_ERR_INVALID_ARG),
    (dict(d=48), fa.FA_ERR_UNSUPPORTED),
    (dict(v=A + 8), fa.FA_ERR_MISALIGNED),
])
def test_gqa_rejects(kw, code):
    assert fwd_gqa(**kw) == code
    assert fa.fa_last_error() != ""
    assert bwd_gqa(**kw) == code


def test_gqa_bwd_rejects_small_workspace():
    need = fa.fa_bwd_gqa_workspace_size(1, 4, 2, 128, 64)
    assert bwd_gqa(workspace_bytes=need - 16) == fa.FA_ERR_WORKSPACE
    # the plain backward's workspace lacks the two fp32 dK, dV accumulators
    assert bwd_gqa(workspace_bytes=fa.fa_bwd_workspace_size(1, 4, 128, 64)) == fa.FA_ERR_WORKSPACE


def test_gqa_workspace_size():
    base = fa.fa_bwd_workspace_size(2, 8, 1000, 128)
    assert fa.fa_bwd_gqa_workspace_size(2, 8, 8, 1000, 128) == base
    acc = -(-2 * 2 * 1000 * 128 * 4 // 256) * 256
    assert fa.fa_bwd_gqa_workspace_size(2, 8, 2, 1000, 128) == base + 2 * acc
    assert fa.fa_bwd_gqa_workspace_size(2, 8, 3, 1000, 128) == 0
    assert fa.fa_bwd_gqa_workspace_size(2, 8, 0, 1000, 128) == 0


def fwd_split(**kw):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=4, H_kv=2, Nq=4, Nk=1000, d=128, causal=1,
             scale=0.125, splits=4, workspace=A, workspace_bytes=1 << 30, stream=None)
    a.update(kw)
    return fa.fa_fwd_splitkv(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(splits=0), fa.FA_ERR_INVALID_ARG),
    (dict(splits=-3), fa.FA_ERR_INVALID_ARG),
    (dict(Nq=2000), fa.FA_ERR_INVALID_ARG),          # causal with more queries than keys
    (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
    (dict(Nk=0), fa.FA_ERR_INVALID_ARG),
    (dict(H_kv=3), fa.FA_ERR_INVALID_ARG),
    (dict(d=80), fa.FA_ERR_UNSUPPORTED),
    (dict(k=A + 4), fa.FA_ERR_MISALIGNED),
    (dict(workspace=None), fa.FA_ERR_WORKSPACE),
    (dict(workspace_bytes=64), fa.FA_ERR_WORKSPACE),
])
def test_splitkv_rejects(kw, code):
    assert fwd_split(**kw) == code
    assert fa.fa_last_error() != ""


def test_splitkv_workspace_size():
    # Nk = 1000 -> 8 key tiles; 4 splits of 2 tiles: 4 fp32 partial rows of d plus 4 logsumexps
    rows = 1 * 4 * 4
    want = -(-4 * rows * 128 * 4 // 256) * 256 + -(-4 * rows * 4 // 256) * 256
    assert fa.fa_fwd_splitkv_workspace_size(1, 4, 4, 1000, 128, 4) == want
    # requests beyond the tile count are reduced to it; one range needs no workspace
    assert fa.fa_fwd_splitkv_workspace_size(1, 4, 4, 1000, 128, 100) == \
        fa.fa_fwd_splitkv_workspace_size(1, 4, 4, 1000, 128, 8)
    assert fa.fa_fwd_splitkv_workspace_size(1, 4, 4, 100, 128, 4) == 0
    assert fa.fa_fwd_splitkv_workspace_size(1, 4, 4, 1000, 128, 1) == 0
    # 3 requested ranges over 8 tiles: chunks of 3 tiles -> 3 non-empty ranges
    assert fa.fa_fwd_splitkv_workspace_size(1, 1, 1, 1000, 64, 3) == \
        -(-3 * 64 * 4 // 256) * 256 + 256
    assert fa.fa_fwd_splitkv_workspace_size(0, 4, 4, 1000, 128, 4) == 0


def test_splitkv_one_range_needs_no_workspace():
    # a single key tile: nothing to merge, so a null workspace is fine (fails later: no device)
    rc = fwd_split(Nk=100, Nq=4, workspace=None, workspace_bytes=0)
    assert rc not in (fa.FA_ERR_WORKSPACE, fa.FA_ERR_INVALID_ARG)


def host_call(**kw):
    a = dict(q=A, k=A, v=A, dO=A, o=None, lse=None, dq=A, dk=A, dv=A, B=2, H=3, N=256, d=128,
             causal=1, scale=0.125, chunks=2, device_buffer=1 << 30, device_bytes=1 << 40,
             stream=None)
    a.update(kw)
    return fa.fa_fwd_bwd_host(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(chunks=0), fa.FA_ERR_INVALID_ARG),
    (dict(chunks=7), fa.FA_ERR_INVALID_ARG),        # more chunks than B*H heads
    (dict(q=None), fa.FA_ERR_INVALID_ARG),
    (dict(dv=None), fa.FA_ERR_INVALID_ARG),
    (dict(d=72), fa.FA_ERR_UNSUPPORTED),
    (dict(device_buffer=None), fa.FA_ERR_WORKSPACE),
    (dict(device_buffer=(1 << 30) + 128), fa.FA_ERR_WORKSPACE),
    (dict(device_bytes=4096), fa.FA_ERR_WORKSPACE),
])
def test_host_pipeline_rejects(kw, code):
    assert host_call(**kw) == code
    assert fa.fa_last_error() != ""


def test_host_pipeline_device_bytes():
    B, H, N, d = 2, 16, 8192, 128
    t = B * H * N * d * 2
    one = fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, 1)
    four = fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, 4)
    # eight full-size tensors and L, plus one chunk's backward workspace
    assert one == 8 * t + B * H * N * 4 + fa.fa_bwd_workspace_size(B, H, N, d)
    assert four == 8 * t + B * H * N * 4 + fa.fa_bwd_workspace_size(1, 8, N, d)
    assert fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, 0) == 0
    assert fa.fa_fwd_bwd_host_device_bytes(B, H, N, d, 33) == 0
