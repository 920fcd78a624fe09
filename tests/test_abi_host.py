"""Host-side checks of the C ABI (no GPU needed, no device memory touched).

The shared library must load and export every function include/svdq.h
declares; sizes, layouts and argument validation are pure host logic.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from w4a4_rank_corrected_act_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "svdq.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = svdq.lib()
    names = _declared_functions()
    assert len(names) >= 19
    for n in names:
        assert hasattr(lib, n), n
        assert n in binding.SIGNATURES, f"binding lacks {n}"
    assert "sm_100a" in svdq.svdq_version()


def test_status_strings():
    for code, name in binding.STATUS_NAMES.items():
        assert svdq.svdq_status_string(code) == name


def test_sizes():
    assert svdq.svdq_act_codes_bytes(4608, 3072) == 4608 * 1536
    assert svdq.svdq_act_scales_bytes(4608, 3072) == 4608 * 192
    assert svdq.svdq_act_scales_bytes(16, 3072) == 128 * 192          # rows padded to 128
    assert svdq.svdq_act_scales_bytes(0, 3072) == 0
    al = lambda x: (x + 255) // 256 * 256                              # noqa: E731
    M, N, K, r = 4608, 9216, 3072, 32
    mp = (M + 127) // 128 * 128
    partials = al(8 * mp * r * 4) + al(mp // 128 * 8 * 8)
    assert svdq.svdq_forward_workspace_bytes(M, N, K, r) == (al(M * K // 2) + al(M * K // 16) + al(M * r * 2)
                                                             + partials)
    assert svdq.svdq_act_workspace_bytes(M, K, r) == partials
    assert svdq.svdq_act_workspace_bytes(M, K, 0) == 256
    wb = (al(N * K // 2) + al(N * K // 16) + al(K * r * 2) + al(K * r * 2) + al(N * r * 2)
          + al(K * 4) + al(N * 2) + al(K * r * 2))
    assert svdq.svdq_weight_bytes(N, K, r, 1) == wb
    assert svdq.svdq_weight_bytes(N, K, r, 0) == wb - al(N * 2)


@pytest.mark.parametrize("N,K,r,ok", [(9216, 3072, 32, True), (128, 256, 0, True),
                                      (100, 3072, 32, False), (256, 3072 + 16, 32, False),
                                      (256, 3072, 12, False), (256, 3072, 72, False),
                                      (128, 256, 136, False), (0, 256, 8, False)])
def test_shape_rules(N, K, r, ok):
    assert (svdq.svdq_weight_bytes(N, K, r, 1) > 0) == ok


def test_weight_bind_carves_aligned_fields():
    N, K, r = 384, 512, 32
    nbytes = svdq.svdq_weight_bytes(N, K, r, 1)
    base = 0x7F0000000000                   # never dereferenced: bind is pointer arithmetic
    w = svdq.svdq_weight_bind(base, nbytes, N, K, r, 1)
    fields = [w.w_codes, w.w_scales, w.L1, w.L1f, w.L2t, w.inv_lambda, w.bias, w.L1t]
    assert all(f % 256 == 0 for f in fields)
    assert fields == sorted(fields) and fields[0] == base
    assert w.L1t + K * r * 2 <= base + nbytes
    assert (w.N, w.K, w.r, w.has_bias) == (N, K, r, 1)
    with pytest.raises(svdq.SvdqError, match="WORKSPACE_TOO_SMALL"):
        svdq.svdq_weight_bind(base, nbytes - 1, N, K, r, 1)
    with pytest.raises(svdq.SvdqError, match="MISALIGNED"):
        svdq.svdq_weight_bind(base + 16, nbytes, N, K, r, 1)
    w0 = svdq.svdq_weight_bind(base, svdq.svdq_weight_bytes(N, K, 0, 0), N, K, 0, 0)
    assert w0.L1 is None and w0.bias is None and w0.L1t is None


def _tile_offset(row, kb16, K):
    """Scale-factor tile layout restated from include/svdq.h."""
    tile = (row // 128) * (K // 64) + kb16 // 4
    return tile * 512 + (row % 32) * 16 + ((row // 32) % 4) * 4 + kb16 % 4


@pytest.mark.parametrize("rows,K", [(1, 64), (130, 256), (256, 3072)])
def test_scale_layout_roundtrip(rows, K):
    rng = np.random.default_rng(rows + K)
    logical = rng.integers(0, 0x7F, (rows, K // 16)).astype(np.uint8)
    mpad = (rows + 127) // 128 * 128
    native = np.full(mpad * K // 16, 0xAA, np.uint8)
    svdq.svdq_scales_to_native(logical.ctypes.data, rows, K, native.ctypes.data)
    for i in range(0, rows, max(1, rows // 17)):
        for j in range(K // 16):
            assert native[_tile_offset(i, j, K)] == logical[i, j]
    # padding rows are zero
    pad = np.ones(mpad * K // 16, bool)
    for i in range(rows):
        for j in range(K // 16):
            pad[_tile_offset(i, j, K)] = False
    assert np.all(native[pad] == 0)
    back = np.empty_like(logical)
    svdq.svdq_scales_to_logical(native.ctypes.data, rows, K, back.ctypes.data)
    assert np.array_equal(back, logical)


def _fake_weight(N=256, K=512, r=32, has_bias=1):
    return svdq.svdq_weight_bind(0x7F0000000000, svdq.svdq_weight_bytes(N, K, r, has_bias), N, K,
                                 r, has_bias)


def test_argument_validation_before_any_device_work():
    w = _fake_weight()
    A = 0x7E0000000000                       # aligned fake device addresses, never touched
    lib = svdq.lib()
    qa = lib.svdq_quantize_act
    W = ctypes.byref(w)
    assert qa(None, 64, W, A, A, A, None) == 1                     # null X
    assert qa(A + 8, 64, W, A, A, A, None) == 3                    # misaligned X
    assert qa(A, -1, W, A, A, A, None) == 1                        # negative M
    assert qa(A, 0, W, A, A, A, None) == 0                         # empty call: no-op
    assert qa(A, 64, W, A, A, None, None) == 1                     # r > 0 needs D
    bad = svdq_weight_copy(w)
    bad.K = 528
    assert qa(A, 64, ctypes.byref(bad), A, A, A, None) == 2        # K % 256 != 0
    bad.K = 500
    assert qa(A, 64, ctypes.byref(bad), A, A, A, None) == 1        # K % 16 != 0
    assert lib.svdq_gemm(A, A, A, 64, W, None, None) == 1
    assert lib.svdq_linear_forward(A, 64, W, A, A, 10, None) == 4  # workspace too small
    assert lib.svdq_linear_forward(A, 0, W, A, A, 0, None) == 0
    nb = svdq.svdq_weight_bytes(256, 512, 32, 1)
    assert lib.svdq_prepare_weight(A, A, None, W, A, nb, None) == 1   # bias iff has_bias
    assert lib.svdq_weight_export(None, None, None, None, None, None, None) == 1


def svdq_weight_copy(w):
    c = binding.svdq_weight()
    ctypes.memmove(ctypes.byref(c), ctypes.byref(w), ctypes.sizeof(w))
    return c


def test_weight_format_field_and_validation():
    N, K, r = 256, 512, 32
    nbytes = svdq.svdq_weight_bytes(N, K, r, 1)
    base = 0x7F0000000000
    assert svdq.svdq_weight_bind(base, nbytes, N, K, r, 1).format == svdq.SVDQ_FORMAT_NVFP4
    w4 = svdq.svdq_weight_bind_format(base, nbytes, N, K, r, 1, svdq.SVDQ_FORMAT_INT4)
    assert w4.format == svdq.SVDQ_FORMAT_INT4
    # the INT4 scale table (N x K/64 fp16) fits in the field before L1
    assert w4.w_scales + N * (K // 64) * 2 <= w4.L1
    with pytest.raises(svdq.SvdqError, match="INVALID_ARG"):
        svdq.svdq_weight_bind_format(base, nbytes, N, K, r, 1, 7)
    lib = svdq.lib()
    A = 0x7E0000000000
    bad = svdq_weight_copy(w4)
    bad.format = 3
    assert lib.svdq_quantize_act(A, 64, ctypes.byref(bad), A, A, A, None) == 1
    assert lib.svdq_gemm(A, A, A, 64, ctypes.byref(bad), A, None) == 1
    # the activation scale buffer covers the INT4 group-major table too
    M = 130
    assert svdq.svdq_act_scales_bytes(M, K) >= ((M + 127) // 128 * 128) * (K // 64) * 2


@pytest.mark.parametrize("rows,rows_pad,K", [(1, 128, 64), (130, 256, 256), (256, 256, 3072)])
def test_int4_scale_layout_roundtrip(rows, rows_pad, K):
    """Group-major fp16 layout restated from include/svdq.h: row i, group g at g * rows_pad + i."""
    rng = np.random.default_rng(rows + K)
    logical = rng.integers(0, 0x7C00, (rows, K // 64)).astype(np.uint16)
    native = np.full(rows_pad * (K // 64), 0xAAAA, np.uint16)
    svdq.svdq_int4_scales_to_native(logical.ctypes.data, rows, rows_pad, K, native.ctypes.data)
    nat2 = native.reshape(K // 64, rows_pad)
    assert np.array_equal(nat2[:, :rows].T, logical)
    assert np.all(nat2[:, rows:] == 0)
    back = np.empty_like(logical)
    svdq.svdq_int4_scales_to_logical(native.ctypes.data, rows, rows_pad, K, back.ctypes.data)
    assert np.array_equal(back, logical)
    with pytest.raises(svdq.SvdqError, match="INVALID_ARG"):
        svdq.svdq_int4_scales_to_logical(native.ctypes.data, rows, rows - 1, K, back.ctypes.data)


def test_act_scales_to_logical_is_the_same_conversion():
    rows, K = 130, 256
    rng = np.random.default_rng(3)
    logical = rng.integers(0, 0x7F, (rows, K // 16)).astype(np.uint8)
    native = np.zeros(((rows + 127) // 128 * 128) * (K // 16), np.uint8)
    svdq.svdq_scales_to_native(logical.ctypes.data, rows, K, native.ctypes.data)
    a = np.empty_like(logical)
    svdq.svdq_act_scales_to_logical(native.ctypes.data, rows, K, a.ctypes.data)
    assert np.array_equal(a, logical)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without the shared library every call raises."""
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="is missing"):
        binding.svdq_weight_bytes(256, 512, 32, 1)
    with pytest.raises(RuntimeError, match="is missing"):
        binding.svdq_version()
