"""GPU parity of the fused MLP pair (svdq_mlp_forward): up-projection, GELU
and the down-projection's activation quantisation in the up-projection's
epilogue, then the down-projection.

Checked against the oracle (oracle/mlp_ref.py, reading R19):
  * H (the kernel's debug output) against bf16(gelu_tanh(Y_up)) evaluated in
    float64 on the up-projection's own bf16 output: equal, or one bf16 step
    apart where the float32 GELU lands on the other side of a rounding
    boundary;
  * the down-projection's NVFP4 codes and E4M3 scales bit-exact, and its D
    within D's bar, against the oracle's activation quantiser run on the
    kernel's H;
  * Y within the output bar against the oracle's down-projection of the
    kernel's H (elements beyond it only through the GPU's D, at most 1 in 10^4).
"""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from oracle import mlp_ref
from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import check_d, check_y, dev_f32, dev_u16, stream, to_np_u16, torch, y_with_d

pytestmark = pytest.mark.gpu


def _align(n):
    return (n + 255) // 256 * 256


def _pair(M, K, F, N, r_up, r_down, seed, bias=True, spec_up=None, spec_down=None):
    t = torch()
    if spec_up is not None:
        du, dd = gen.make_linear(spec_up), gen.make_linear(spec_down)
        X, W1, b1, lam1 = du["X"], du["W"], du["bias"], du["lam"]
        W2, b2 = dd["W"], dd["bias"]
    else:
        rng = np.random.default_rng(seed)
        x = rng.standard_normal((M, K))
        x[:, rng.choice(K, 4, replace=False)] *= 40
        X = gen.to_bf16_bits(x)
        W1 = gen.to_bf16_bits(rng.standard_normal((F, K)) * 0.02)
        W2 = gen.to_bf16_bits(rng.standard_normal((N, F)) * 0.02)
        b1 = gen.to_bf16_bits(rng.standard_normal(F) * 0.01)
        b2 = gen.to_bf16_bits(rng.standard_normal(N) * 0.01)
        lam1 = gen.calibrate_lambda(X, W1)
    if not bias:
        b1 = b2 = None
    up = svdq.SvdqLinear(dev_u16(W1), dev_f32(lam1), dev_u16(b1) if bias else None, r=r_up)
    # the up-projection alone (the general path), and H from it in float64:
    # the down-projection's smoothing factors are calibrated on that H
    Y_up = to_np_u16(up.forward(dev_u16(X).view(t.bfloat16)).view(t.int16))
    H_ref = mlp_ref.mlp_hidden(Y_up)
    lam2 = gen.calibrate_lambda(H_ref, W2)
    down = svdq.SvdqLinear(dev_u16(W2), dev_f32(lam2), dev_u16(b2) if bias else None, r=r_down)
    return X, up, down, Y_up, H_ref, b2


def _run(X, M, up, down):
    t = torch()
    K, F, N = up.K, up.N, down.N
    nb = svdq.svdq_mlp_workspace_bytes(M, K, F, N, up.r, down.r)
    ws = t.zeros(max(nb, 256), dtype=t.uint8, device="cuda")
    Y = t.empty((M, N), dtype=t.int16, device="cuda")
    H = t.empty((M, F), dtype=t.int16, device="cuda")
    Xd = dev_u16(X)
    svdq.svdq_mlp_forward(Xd.data_ptr(), M, up.w, down.w, Y.data_ptr(), H.data_ptr(), ws.data_ptr(), nb, stream())
    t.cuda.synchronize()
    assert svdq.svdq_get_device_status(stream()) == 0
    wsb = ws.cpu().numpy()
    # the down-projection's activation workspace (general layout)
    a = _align(svdq.svdq_forward_workspace_bytes(M, F, K, up.r))
    codes = wsb[a:a + M * F // 2].reshape(M, F // 2)
    s0 = a + _align(M * F // 2)
    nsc = svdq.svdq_act_scales_bytes(M, F)
    native = np.ascontiguousarray(wsb[s0:s0 + nsc])
    scales = np.empty((M, F // 16), np.uint8)
    svdq.svdq_scales_to_logical(native.ctypes.data, M, F, scales.ctypes.data)
    d0 = s0 + _align(nsc)
    D = wsb[d0:d0 + M * down.r * 2].view(np.uint16).reshape(M, down.r) if down.r else None
    return to_np_u16(Y), to_np_u16(H), codes, scales, D


def _check(X, M, up, down, Y_up, H_ref, b2, name, rows=None):
    Y, H, codes, scales, D = _run(X, M, up, down)
    # H: one bf16 step of the float64 value at most
    hg, ho = ref.bf16_to_f64(H), ref.bf16_to_f64(H_ref)
    step = np.abs(H.astype(np.int32) - H_ref.astype(np.int32))
    same_sign = np.signbit(hg) == np.signbit(ho)
    ok = (step <= 1) & same_sign | (hg == ho)
    if not np.all(ok):
        idx = np.argwhere(~ok)[:8]
        yv = ref.bf16_to_f64(Y_up)
        rows_ = [(int(i), int(j), float(yv[i, j]), float(hg[i, j]), float(ho[i, j])) for i, j in idx]
        raise AssertionError(f"{name}: H off by more than one bf16 step at {int((~ok).sum())} elements; "
                             f"(m, n, Y_up, H_gpu, H_ref): {rows_}")
    print(f"{name}: H differs from the float64 GELU by one bf16 step at {int((H != H_ref).sum())} of {H.size}")
    exp = down.export()
    if rows is None:
        rows = np.arange(M)
    xo = ref.quantize_act(H[rows], exp["inv_lambda"], exp["L1"] if down.r else None)
    assert int((codes[rows] != xo["x_codes"]).sum()) == 0, f"{name}: hidden codes"
    assert np.array_equal(scales[rows], xo["x_scales"]), f"{name}: hidden scales"
    yd = None
    if down.r:
        check_d(D[rows], xo["D"], xo["D_abs"])
    prep = dict(inv_lambda=exp["inv_lambda"], L1=exp["L1"], L2t=exp["L2t"], w_codes=exp["w_codes"],
                w_scales=exp["w_scales"], bias=b2)
    o = ref.linear_forward(H, prep, rows=None if len(rows) == M else rows)
    if down.r:
        yd = y_with_d(o["Y64"], o["D"], D[rows], exp["L2t"])
    return check_y(Y[rows], o["Y64"], name, y_given_gpu_d=yd)


@pytest.mark.parametrize("M,K,F,N,r_up,r_down,bias", [(300, 512, 768, 384, 32, 16, True),
                                                       (129, 768, 1024, 512, 16, 32, False),
                                                       (40, 256, 512, 256, 0, 8, True),
                                                       (700, 1024, 2048, 768, 32, 0, True),
                                                       (16, 512, 1024, 256, 32, 32, True)])
def test_mlp_pair_parity(M, K, F, N, r_up, r_down, bias):
    X, up, down, Y_up, H_ref, b2 = _pair(M, K, F, N, r_up, r_down, seed=M + K + F + N, bias=bias)
    _check(X, M, up, down, Y_up, H_ref, b2, f"mlp {M}x{K}x{F}x{N}")


def test_mlp_pair_parity_tensor_core_activation_kernel():
    """The pair with the up-projection's activation kernel forced to the 128-row
    kernel (D on the tensor cores, K split with float32 partials)."""
    with svdq.override(svdq.SVDQ_OVERRIDE_ACT_KERNEL, 2):
        X, up, down, Y_up, H_ref, b2 = _pair(300, 1536, 1024, 512, 32, 32, seed=31, bias=True)
        _check(X, 300, up, down, Y_up, H_ref, b2, "mlp (128-row activation kernel)")


def test_mlp_pair_matches_the_unfused_pair():
    """The fused pair against the same two layers run one after the other
    (svdq_linear_forward, GELU of the bf16 output in float64, svdq_linear_forward)."""
    t = torch()
    M, K, F, N = 256, 512, 1024, 512
    X, up, down, Y_up, H_ref, b2 = _pair(M, K, F, N, 32, 32, seed=9)
    Y, H, *_ = _run(X, M, up, down)
    Y2 = to_np_u16(down.forward(dev_u16(H_ref).view(t.bfloat16)).view(t.int16))
    a, b = ref.bf16_to_f64(Y), ref.bf16_to_f64(Y2)
    rms = float(np.sqrt(np.mean(b ** 2)))
    # H may differ by one bf16 step, which moves Y by at most that step through W_down
    assert np.max(np.abs(a - b)) <= 2e-2 * rms


def test_mlp_pair_workload_full_size():
    """The MLP pair at 1024 x 1024: M = 4608, K = 3072, F = 12288, N = 3072, r = 32
    (sampled rows against the oracle; every row is independent)."""
    su, sd = gen.workload("mlp_up"), gen.workload("mlp_down")
    X, up, down, Y_up, H_ref, b2 = _pair(su.M, su.K, su.N, sd.N, su.r, sd.r, seed=0, spec_up=su, spec_down=sd)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, su.M - 1], rng.choice(su.M, 62, replace=False)]))
    _check(X, su.M, up, down, Y_up, H_ref, b2, "mlp pair (config 3)", rows=rows)
