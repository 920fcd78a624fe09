"""GPU parity of the few-token path (M <= 32): the activation kernel that
splits K over CTAs and the swapped-operand block-scaled GEMM, through
svdq_linear_forward (and its head-major and no-allocation variants).

Checked against the oracle: the activation codes and E4M3 scales bit-exact
(read from the workspace, whose few-token layout the header documents), the
sum of the D partials within D's bar, and Y within the output bar; the same
calls with the path turned off (SVDQ_OVERRIDE_SMALL_M = 1) agree with it."""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import (check_d, check_y, dev_f32, dev_u16, stream, to_np_u16, torch, y_with_d)

pytestmark = pytest.mark.gpu


def _layer(M, K, N, r, seed, bias=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    x[:, rng.choice(K, 4, replace=False)] *= 40
    w = rng.standard_normal((N, K)) * 0.02
    w[:, rng.choice(K, 2, replace=False)] *= 10
    X, W = gen.to_bf16_bits(x), gen.to_bf16_bits(w)
    B = gen.to_bf16_bits(rng.standard_normal(N) * 0.01) if bias else None
    lam = gen.calibrate_lambda(X, W)
    lin = svdq.SvdqLinear(dev_u16(W), dev_f32(lam), dev_u16(B) if bias else None, r=r)
    return lin, X, B


def _align(n):
    return (n + 255) // 256 * 256


def _small_ws_fields(ws_bytes_np, M, K, r):
    """codes [M][K/2], scale words [K/64][32], float32 partials [K/256][M][r]."""
    c = _align(M * K // 2)
    s = _align(K // 64 * 32 * 4)
    codes = ws_bytes_np[: M * K // 2].reshape(M, K // 2)
    words = ws_bytes_np[c:c + K // 64 * 32 * 4].view(np.uint32).reshape(K // 64, 32)
    dpart = ws_bytes_np[c + s:c + s + (K // 256) * M * r * 4].view(np.float32).reshape(K // 256, M, r)
    return codes, words, dpart


def _d_of_partials(dpart):
    """bf16 of the float32 sum of the partials in slice order (the GEMM's own order)."""
    acc = np.zeros(dpart.shape[1:], np.float32)
    for s in range(dpart.shape[0]):
        acc = (acc + dpart[s]).astype(np.float32)
    return ref.f64_to_bf16(acc.astype(np.float64))


def _forward(lin, X, M, head_dim=0):
    t = torch()
    nb = lin.workspace_bytes(M)
    ws = t.zeros(max(nb, 256), dtype=t.uint8, device="cuda")
    Xd = dev_u16(X)
    if head_dim:
        Y = t.empty((lin.N // head_dim, M, head_dim), dtype=t.int16, device="cuda")
        svdq.svdq_linear_forward_heads(Xd.data_ptr(), M, lin.w, head_dim, Y.data_ptr(), ws.data_ptr(), nb,
                                       stream())
    else:
        Y = t.empty((M, lin.N), dtype=t.int16, device="cuda")
        svdq.svdq_linear_forward(Xd.data_ptr(), M, lin.w, Y.data_ptr(), ws.data_ptr(), nb, stream())
    t.cuda.synchronize()
    return to_np_u16(Y), ws.cpu().numpy()


@pytest.mark.parametrize("M,K,N,r,bias", [(1, 3072, 18432, 32, True), (15, 3072, 18432, 32, True),
                                          (16, 3072, 18432, 32, True), (17, 3072, 2048, 32, True),
                                          (32, 3072, 4096, 32, False), (9, 256, 1024, 16, True),
                                          (24, 768, 640, 64, True), (5, 3840, 512, 8, True),
                                          (32, 1024, 384, 0, True), (3, 512, 128, 48, False)])
def test_small_m_forward_parity(M, K, N, r, bias):
    lin, X, B = _layer(M, K, N, r, seed=M * 31 + K + N + r, bias=bias)
    exp = lin.export()
    Y, wsb = _forward(lin, X, M)
    assert svdq.svdq_get_device_status(stream()) == 0
    inv = exp["inv_lambda"]
    xo = ref.quantize_act(X, inv, exp["L1"] if r else None)
    codes, words, dpart = _small_ws_fields(wsb, M, K, r)
    assert int((codes != xo["x_codes"]).sum()) == 0, "activation codes"
    # scale word j of token m holds the scales of 16-column blocks 4 j .. 4 j + 3
    sc = words[:, :M].T.copy().view(np.uint8).reshape(M, K // 16)
    assert np.array_equal(sc, xo["x_scales"]), "activation scales"
    assert np.all(words[:, M:] == 0), "scale words of padding tokens"
    Dg = None
    if r:
        Dg = _d_of_partials(dpart)
        check_d(Dg, xo["D"], xo["D_abs"])
    prep = dict(inv_lambda=inv, L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=B)
    o = ref.linear_forward(X, prep)
    yd = y_with_d(o["Y64"], o["D"], Dg, exp["L2t"]) if r else None
    check_y(Y, o["Y64"], f"small-M {M}x{K}x{N} r={r}", y_given_gpu_d=yd)


def test_small_m_matches_the_general_path():
    """The same layer with the few-token path switched off (the 128-row
    GEMM) gives the same Y up to float32 summation order."""
    M, K, N, r = 16, 3072, 4608, 32
    lin, X, B = _layer(M, K, N, r, seed=4)
    Ys, _ = _forward(lin, X, M)
    with svdq.override(svdq.SVDQ_OVERRIDE_SMALL_M, 1):
        Yg, _ = _forward(lin, X, M)
    a, b = ref.bf16_to_f64(Ys), ref.bf16_to_f64(Yg)
    rms = float(np.sqrt(np.mean(b ** 2)))
    assert np.all(np.abs(a - b) <= 4e-3 * rms + 2 * np.abs(b) * 2.0 ** -7)


@pytest.mark.parametrize("hd", [64, 128])
def test_small_m_heads(hd):
    M, K, N, r = 20, 1024, 1536, 32
    lin, X, _ = _layer(M, K, N, r, seed=hd)
    Yr, _ = _forward(lin, X, M)
    Yh, _ = _forward(lin, X, M, head_dim=hd)
    assert np.array_equal(Yh, np.ascontiguousarray(Yr.reshape(M, N // hd, hd).transpose(1, 0, 2)))


def test_small_m_workload_full_size():
    """The small-M workload itself (M = 16, K = 3072, N = 18432, r = 32)."""
    spec = gen.workload("small_m")
    d = gen.make_linear(spec)
    lin = svdq.SvdqLinear(dev_u16(d["W"]), dev_f32(d["lam"]), dev_u16(d["bias"]), r=spec.r)
    exp = lin.export()
    Y, wsb = _forward(lin, d["X"], spec.M)
    xo = ref.quantize_act(d["X"], exp["inv_lambda"], exp["L1"])
    codes, words, dpart = _small_ws_fields(wsb, spec.M, spec.K, spec.r)
    assert int((codes != xo["x_codes"]).sum()) == 0
    Dg = _d_of_partials(dpart)
    check_d(Dg, xo["D"], xo["D_abs"])
    prep = dict(inv_lambda=exp["inv_lambda"], L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=d["bias"])
    o = ref.linear_forward(d["X"], prep)
    check_y(Y, o["Y64"], "small_m", y_given_gpu_d=y_with_d(o["Y64"], o["D"], Dg, exp["L2t"]))
