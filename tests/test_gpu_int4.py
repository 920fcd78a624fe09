"""GPU parity of the INT4 variant of the layer against its oracle (oracle/int4_ref.py),
through the C ABI.

Bars, as for NVFP4: INT4 codes and fp16 group scales bit-exact (activations and,
given the library's exported bf16 factors, the weight); D within 1 bf16 ulp plus
the float32 accumulation bound; Y within 4e-3 rms(Y_oracle) + 2 bf16 ulps.  The
INT4 GEMM forms each group's integer sum exactly, so its only departures from
the oracle's float64 sum are the float32 scaling and accumulation.
"""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from oracle import int4_ref as i4
from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import (check_d, check_y, dev_f32, gpu_d, y_with_d, dev_u16, dev_u8, empty_u8,
                      stream, to_np_u16, torch)

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, seed, outliers=4, scale=40.0, wcols=2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    if outliers:
        x[:, rng.choice(K, outliers, replace=False)] *= scale
    w = rng.standard_normal((N, K)) * 0.02
    if wcols:
        w[:, rng.choice(K, wcols, replace=False)] *= 10
    b = rng.standard_normal(N) * 0.01
    X, W, B = gen.to_bf16_bits(x), gen.to_bf16_bits(w), gen.to_bf16_bits(b)
    return X, W, B, gen.calibrate_lambda(X, W)


def _prepare(W, lam, bias, r):
    t = torch()
    lin = svdq.SvdqLinear(dev_u16(W), dev_f32(lam), dev_u16(bias) if bias is not None else None, r=r,
                          format="int4")
    t.cuda.synchronize()
    return lin, lin.export()


def _oracle_prep_from_export(W, lam, bias, exp, r):
    inv = ref.inv_lambda_of(lam)
    assert np.array_equal(exp["inv_lambda"].view(np.uint32), inv.view(np.uint32)), "inv_lambda"
    K, N = W.shape[1], W.shape[0]
    L1 = exp["L1"] if r else np.zeros((K, 0), np.uint16)
    L2t = exp["L2t"] if r else np.zeros((N, 0), np.uint16)
    _, codes, scales = i4.residual_quantize_int4(ref.smooth_weight(W, lam), L1, np.ascontiguousarray(L2t.T))
    nbad = int((codes != exp["w_codes"]).sum())
    assert nbad == 0, f"INT4 weight codes differ in {nbad} bytes"
    assert np.array_equal(scales, exp["w_scales"]), "INT4 weight scales differ"
    return dict(inv_lambda=inv, L1=L1, L2t=L2t, w_codes=codes, w_scales=scales, bias=bias)


def _act_scales_logical(scales_dev, M, K):
    mpad = (M + 127) // 128 * 128
    nat = scales_dev[: mpad * (K // 64) * 2].cpu().numpy().view(np.uint16).copy()
    logical = np.empty((M, K // 64), np.uint16)
    svdq.svdq_int4_scales_to_logical(nat.ctypes.data, M, mpad, K, logical.ctypes.data)
    return logical, nat.reshape(K // 64, mpad)


def _run_act(X, lin):
    t = torch()
    M, K = X.shape
    Xd = dev_u16(X)
    codes = empty_u8(svdq.svdq_act_codes_bytes(M, K))
    scales = t.full((max(svdq.svdq_act_scales_bytes(M, K), 256),), 0x5A, dtype=t.uint8, device="cuda")
    D = t.empty((max(M, 1), max(lin.r, 1)), dtype=t.int16, device="cuda")
    svdq.svdq_quantize_act(Xd.data_ptr(), M, lin.w, codes.data_ptr(), scales.data_ptr(),
                           D.data_ptr() if lin.r else 0, stream())
    t.cuda.synchronize()
    c = codes[: M * K // 2].cpu().numpy().reshape(M, K // 2)
    logical, native = _act_scales_logical(scales, M, K)
    d = D.cpu().numpy().view(np.uint16)[:M, :lin.r] if lin.r else None
    return c, logical, native, d


@pytest.mark.parametrize("M,K,N,r", [(256, 512, 128, 32), (1, 256, 128, 16), (17, 768, 128, 32),
                                     (129, 512, 128, 64), (300, 1024, 256, 8), (64, 256, 128, 0)])
def test_int4_act_parity(M, K, N, r):
    X, W, B, lam = _inputs(M, K, N, seed=M * 5 + K + r)
    lin, exp = _prepare(W, lam, None, r)
    codes, scales, native, d = _run_act(X, lin)
    o = i4.quantize_act_int4(X, ref.inv_lambda_of(lam), exp["L1"] if r else None)
    nbad = int((codes != o["x_codes"]).sum())
    assert nbad == 0, f"{nbad} INT4 code bytes differ"
    assert np.array_equal(scales, o["x_scales"])
    assert np.all(native[:, M:] == 0), "padding rows of the scale table must be zero"
    if r:
        check_d(d, o["D"], o["D_abs"])


def test_int4_act_rounding_cases():
    """Half-way quotients, saturated and zero groups (lambda = 1, s = amax / 7)."""
    K, N = 256, 128
    base = [7.0, 0.5, 1.5, 2.5, 3.5, 4.5, 5.5, 6.5, -0.5, -1.5, -2.5, -3.5, -6.5, -7.0, 0.0, -0.0]
    rows = [[v * 2.0 ** k for v in base] * (K // 16) for k in range(-8, 9, 2)]
    rows.append(([1e6, -1e6] + [1.0] * 14) * (K // 16))            # saturated scale: clamp to 7 / -8
    rows.append([0.0] * K)                                            # zero groups
    rows.append(([3e-8, -1e-8] + [0.0] * 14) * (K // 16))            # amax / 7 below fp16 range
    rows.append(([7.0, 0.4999, 0.5001, 2.4999, 2.5001, 6.4999, 6.5001, -3.5001] * 2) * (K // 16))
    X = gen.to_bf16_bits(np.array(rows, dtype=np.float64))
    lam = np.ones(K, np.float32)
    W = gen.to_bf16_bits(np.random.default_rng(0).standard_normal((N, K)) * 0.02)
    lin, _ = _prepare(W, lam, None, 0)
    codes, scales, _, _ = _run_act(X, lin)
    o = i4.quantize_act_int4(X, np.ones(K, np.float32), None)
    assert np.array_equal(scales, o["x_scales"])
    assert np.array_equal(codes, o["x_codes"]), np.argwhere(codes != o["x_codes"])[:8]


def test_int4_act_random_lambda_sweep():
    rng = np.random.default_rng(78)
    M, K, N = 512, 2048, 128
    x = rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 6, (M, 1)))
    X = gen.to_bf16_bits(x)
    W = gen.to_bf16_bits(rng.standard_normal((N, K)) * 0.02)
    lam = np.exp(rng.uniform(-3, 3, K)).astype(np.float32)
    lin, _ = _prepare(W, lam, None, 0)
    codes, scales, _, _ = _run_act(X, lin)
    o = i4.quantize_act_int4(X, ref.inv_lambda_of(lam), None)
    assert np.array_equal(scales, o["x_scales"])
    assert int((codes != o["x_codes"]).sum()) == 0


@pytest.mark.parametrize("N,K,r,with_bias", [(512, 512, 32, True), (256, 1024, 16, False),
                                             (384, 768, 0, True), (128, 256, 8, False)])
def test_int4_prepare_parity(N, K, r, with_bias):
    _, W, B, lam = _inputs(64, K, N, seed=N + K + r + 1)
    _prepare_and_check(W, lam, B if with_bias else None, r)


def _prepare_and_check(W, lam, bias, r):
    lin, exp = _prepare(W, lam, bias, r)
    return lin, exp, _oracle_prep_from_export(W, lam, bias, exp, r)


@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 32), (1, 256, 128, 16), (129, 768, 384, 32),
                                     (300, 1024, 256, 0), (64, 512, 1024, 64), (513, 256, 640, 8)])
def test_int4_gemm_parity(M, K, N, r):
    """svdq_gemm with an INT4 weight on oracle-produced activation codes."""
    t = torch()
    X, W, B, lam = _inputs(M, K, N, seed=3 * M + K + N + r + 7)
    lin, exp, prep = _prepare_and_check(W, lam, B, r)
    o = i4.linear_forward_int4(X, prep)
    codes = dev_u8(o["x_codes"])
    mpad = (M + 127) // 128 * 128
    logical = np.ascontiguousarray(o["x_scales"])
    native = np.zeros(max(svdq.svdq_act_scales_bytes(M, K) // 2, 128), np.uint16)
    svdq.svdq_int4_scales_to_native(logical.ctypes.data, M, mpad, K, native.ctypes.data)
    sc = t.from_numpy(native.view(np.int16)).cuda()
    D = dev_u16(o["D"]) if r else None
    Y = t.empty((M, N), dtype=t.int16, device="cuda")
    svdq.svdq_gemm(codes.data_ptr(), sc.data_ptr(), D.data_ptr() if r else 0, M, lin.w, Y.data_ptr(), stream())
    t.cuda.synchronize()
    check_y(to_np_u16(Y), o["Y64"], "int4 gemm")
    assert svdq.svdq_get_device_status(stream()) == 0


def test_int4_gemm_extreme_group_sums():
    """Codes at the ends of the range: group sums up to 64 * 49 with codes +-7,
    then 64 * 56 with saturated activation scales (codes 7 and -8); the integer
    sums (|c| <= 4096) must stay exact through the float conversion."""
    t = torch()
    M, K, N = 128, 256, 128
    rng = np.random.default_rng(3)
    signs = rng.choice([-1.0, 1.0], size=(M, K))
    x = 7.0 * signs
    x[:, ::64] = 7.0                      # amax 7 in every group -> s = 1
    X = gen.to_bf16_bits(x)
    w = 0.07 * rng.choice([-1.0, 1.0], size=(N, K))
    W = gen.to_bf16_bits(w)
    lam = np.ones(K, np.float32)
    lin, exp, prep = _prepare_and_check(W, lam, None, 0)
    o = i4.linear_forward_int4(X, prep)
    Xd = dev_u16(X)
    Y = lin.forward(Xd.view(t.bfloat16))
    t.cuda.synchronize()
    check_y(to_np_u16(Y.view(t.int16)), o["Y64"], "int4 extreme")
    # saturated groups: codes -8 next to 7
    x2 = np.where(rng.random((M, K)) < 0.5, 1e6, -1e6)
    X2 = gen.to_bf16_bits(x2)
    o2 = i4.linear_forward_int4(X2, prep)
    Y2 = lin.forward(dev_u16(X2).view(t.bfloat16))
    t.cuda.synchronize()
    check_y(to_np_u16(Y2.view(t.int16)), o2["Y64"], "int4 saturated")


@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 32), (700, 1280, 768, 48), (37, 3072, 384, 32)])
def test_int4_forward_parity(M, K, N, r):
    """The whole layer (svdq_linear_forward) with an INT4 weight."""
    t = torch()
    X, W, B, lam = _inputs(M, K, N, seed=11 * M + K + r)
    lin, exp, prep = _prepare_and_check(W, lam, B, r)
    Y = lin.forward(dev_u16(X).view(t.bfloat16))
    t.cuda.synchronize()
    o = i4.linear_forward_int4(X, prep)
    yd = y_with_d(o["Y64"], o["D"], gpu_d(lin, dev_u16(X), M), exp["L2t"]) if r else None
    check_y(to_np_u16(Y.view(t.int16)), o["Y64"], "int4 forward", y_given_gpu_d=yd)


def test_int4_heads_match_row_major():
    t = torch()
    M, K, N, r, hd = 200, 512, 384, 32, 64
    X, W, B, lam = _inputs(M, K, N, seed=99)
    lin, _ = _prepare(W, lam, B, r)
    Xd = dev_u16(X)
    Y = lin.forward(Xd.view(t.bfloat16))
    Yh = t.empty((N // hd, M, hd), dtype=t.int16, device="cuda")
    ws = empty_u8(lin.workspace_bytes(M))
    svdq.svdq_linear_forward_heads(Xd.data_ptr(), M, lin.w, hd, Yh.data_ptr(), ws.data_ptr(),
                                   lin.workspace_bytes(M), stream())
    t.cuda.synchronize()
    yr = to_np_u16(Y.view(t.int16))
    yh = to_np_u16(Yh)
    assert np.array_equal(yh.transpose(1, 0, 2).reshape(M, N), yr)


def test_int4_export_import_and_file_round_trip(tmp_path):
    t = torch()
    M, K, N, r = 130, 512, 256, 16
    X, W, B, lam = _inputs(M, K, N, seed=5)
    lin, exp = _prepare(W, lam, B, r)
    Xd = dev_u16(X).view(t.bfloat16)
    Y0 = lin.forward(Xd)
    lin2 = svdq.SvdqLinear.from_export(exp, bias=B)       # format implied by the fp16 scales
    assert lin2.format == "int4"
    path = tmp_path / "w_int4.npz"
    lin.save(path)
    lin3 = svdq.SvdqLinear.load(path)
    assert lin3.format == "int4"
    Y2, Y3 = lin2.forward(Xd), lin3.forward(Xd)
    t.cuda.synchronize()
    assert t.equal(Y0.view(t.int16), Y2.view(t.int16))
    assert t.equal(Y0.view(t.int16), Y3.view(t.int16))


def test_int4_full_size_sampled():
    """The qkv workload's shape (M=4608, K=3072, N=9216, r=32) in INT4: sampled
    weight rows and token rows checked exactly against the oracle."""
    t = torch()
    spec = gen.workload("qkv")
    d = gen.make_linear(spec)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    lin = svdq.SvdqLinear(dev_u16(d["W"]), dev_f32(d["lam"]), dev_u16(d["bias"]), r=r, format="int4")
    exp = lin.export()
    inv = ref.inv_lambda_of(d["lam"])
    rng = np.random.default_rng(4)
    wrows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 64, replace=False)]))
    _, wc, ws = i4.residual_quantize_int4(ref.smooth_weight(d["W"][wrows], d["lam"]), exp["L1"],
                                          np.ascontiguousarray(exp["L2t"][wrows].T))
    assert int((wc != exp["w_codes"][wrows]).sum()) == 0
    assert np.array_equal(ws, exp["w_scales"][wrows])
    X = dev_u16(d["X"])
    Y = lin.forward(X.view(t.bfloat16))
    t.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 48, replace=False)]))
    prep = dict(inv_lambda=inv, L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=d["bias"])
    o = i4.linear_forward_int4(d["X"], prep, rows=rows)
    yd = y_with_d(o["Y64"], o["D"], gpu_d(lin, X, M)[rows], exp["L2t"])
    check_y(to_np_u16(Y.view(t.int16))[rows], o["Y64"], "int4 qkv", y_given_gpu_d=yd)
    assert svdq.svdq_get_device_status(stream()) == 0


@pytest.mark.parametrize("M", [200, 2600])
def test_int4_host_buffers_and_noalloc_match_device_path(M):
    """The host-buffer path (chunked above 1024 rows) and the no-allocation path
    run the same INT4 kernels: their outputs equal the workspace path's bit for bit."""
    t = torch()
    K, N, r = 512, 384, 32
    X, W, B, lam = _inputs(M, K, N, seed=95)
    lin, _ = _prepare(W, lam, B, r)
    Yd = to_np_u16(lin.forward(dev_u16(X).view(t.bfloat16)).view(t.int16))
    Xh = t.from_numpy(X.view(np.int16).copy()).pin_memory()
    Yh = t.empty((M, N), dtype=t.int16).pin_memory()
    Xdev = t.empty((M, K), dtype=t.int16, device="cuda")
    Ydev = t.empty((M, N), dtype=t.int16, device="cuda")
    nb = lin.workspace_bytes(M)
    ws = empty_u8(nb)
    t.cuda.synchronize()
    svdq.svdq_linear_forward_host(Xh.data_ptr(), M, lin.w, Yh.data_ptr(), Xdev.data_ptr(),
                                  Ydev.data_ptr(), ws.data_ptr(), nb, stream())
    t.cuda.current_stream().synchronize()
    assert np.array_equal(Yh.numpy().view(np.uint16), Yd)
    Xd = dev_u16(X)
    Yn = t.full((M, N), -1, dtype=t.int16, device="cuda")
    svdq.svdq_linear_forward_noalloc(Xd.data_ptr(), M, lin.w, Yn.data_ptr(), stream())
    t.cuda.synchronize()
    assert np.array_equal(to_np_u16(Yn), Yd)
