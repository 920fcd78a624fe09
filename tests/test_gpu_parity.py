"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Bars:
  * activation and weight NVFP4 codes and E4M3 scales: bit-exact;
  * inv_lambda: bit-exact;
  * D: 1 bf16 ulp + 2^-14 * sum|Xhat L1| (float32 accumulation bound);
  * Y: every element within 4e-3 rms(Y_oracle) + 2 bf16 ulps of itself; the oracle
    runs end to end (its own activation codes, scales and D) on the library's
    own exported weight; nothing else is added to that bar;
  * the rank-r factors: ||L1 L2 - L1o L2o||_F <= 1e-2 ||L1o L2o||_F against the
    oracle's own SVD (bf16 storage of both sides limits this to ~2e-3).
"""
import numpy as np
import pytest

import w4a4_rank_corrected_act_b200 as svdq
from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import (check_d, check_y, dev_f32, gpu_d, y_with_d, dev_u16, dev_u8, empty_u8,
                      stream, to_np_u16, torch)

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

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


def _weight_with(K, N, r, inv_lambda, L1=None, has_bias=False):
    """A bound weight whose inv_lambda / L1 fields are filled directly (S1 tests)."""
    t = torch()
    nbytes = svdq.svdq_weight_bytes(N, K, r, int(has_bias))
    buf = t.zeros(nbytes, dtype=t.uint8, device="cuda")
    w = svdq.svdq_weight_bind(buf.data_ptr(), nbytes, N, K, r, int(has_bias))
    base = buf.data_ptr()

    def put(ptr, arr):
        a = np.ascontiguousarray(arr).view(np.uint8).reshape(-1)
        off = ptr - base
        buf[off:off + a.size] = t.from_numpy(a.copy()).cuda()

    put(w.inv_lambda, inv_lambda.astype(np.float32))
    if r:
        put(w.L1, L1.astype(np.uint16))
        put(w.L1f, l1_fragment_order(L1.astype(np.uint16)))
        put(w.L1t, np.ascontiguousarray(L1.astype(np.uint16).T))
    return w, buf


def l1_fragment_order(L1):
    """L1 (K x r) in the B-fragment order documented in include/svdq.h: 32-bit word
    ((g * r/8 + t) * 32 + lane) * 2 + h holds L1[16g + 2(lane%4) + 8h + {0, 1}][8t + lane/4]."""
    K, r = L1.shape
    out = np.zeros(K * r, np.uint16)
    for k in range(K):
        g, kk = divmod(k, 16)
        for j in range(r):
            t, jj = divmod(j, 8)
            lane = jj * 4 + (kk % 8) // 2
            word = ((g * (r // 8) + t) * 32 + lane) * 2 + kk // 8
            out[word * 2 + (k & 1)] = L1[k, j]
    return out


def _run_act(X, inv, L1, N=128, ws=False):
    """Codes, scales and D of X from svdq_quantize_act (ws=False) or from the
    forward's own activation kernel through svdq_quantize_act_ws (ws=True)."""
    M, K = X.shape
    r = 0 if L1 is None else L1.shape[1]
    w, buf = _weight_with(K, N, r, inv, L1)
    t = torch()
    Xd = dev_u16(X)
    codes = empty_u8(svdq.svdq_act_codes_bytes(M, K))
    scales = empty_u8(svdq.svdq_act_scales_bytes(M, K))
    D = t.empty((max(M, 1), max(r, 1)), dtype=t.int16, device="cuda")
    if ws:
        nb = svdq.svdq_act_workspace_bytes(M, K, r)
        wsb = empty_u8(nb)
        with svdq.override(svdq.SVDQ_OVERRIDE_ACT_KERNEL, 2):
            svdq.svdq_quantize_act_ws(Xd.data_ptr(), M, w, codes.data_ptr(), scales.data_ptr(),
                                      D.data_ptr() if r else 0, wsb.data_ptr(), nb, stream())
    else:
        svdq.svdq_quantize_act(Xd.data_ptr(), M, w, codes.data_ptr(), scales.data_ptr(),
                               D.data_ptr() if r else 0, stream())
    t.cuda.synchronize()
    nat = codes[: M * K // 2].cpu().numpy().reshape(M, K // 2)
    sn = scales[: svdq.svdq_act_scales_bytes(M, K)].cpu().numpy()
    logical = np.empty((M, K // 16), np.uint8)
    svdq.svdq_scales_to_logical(sn.ctypes.data, M, K, logical.ctypes.data)
    mpad = (M + 127) // 128 * 128
    full = np.empty((mpad, K // 16), np.uint8)
    svdq.svdq_scales_to_logical(sn.ctypes.data, mpad, K, full.ctypes.data)
    d = D.cpu().numpy().view(np.uint16)[:M, :r] if r else None
    del buf
    return nat, logical, full, d


def _prepare(W, lam, bias, r):
    t = torch()
    lin = svdq.SvdqLinear(dev_u16(W), dev_f32(lam), dev_u16(bias) if bias is not None else None, r=r)
    t.cuda.synchronize()
    return lin, lin.export()


def _oracle_prep_from_export(W, lam, bias, exp, r):
    """Oracle weight built from the library's exported L1/L2 (codes must match)."""
    inv = ref.inv_lambda_of(lam)
    assert np.array_equal(exp["inv_lambda"].view(np.uint32), inv.view(np.uint32)), "inv_lambda"
    w_hat = ref.smooth_weight(W, lam)
    K, N = W.shape[1], W.shape[0]
    L1 = exp["L1"] if r else np.zeros((K, 0), np.uint16)
    L2t = exp["L2t"] if r else np.zeros((N, 0), np.uint16)
    _, codes, scales = ref.residual_quantize(w_hat, L1, np.ascontiguousarray(L2t.T))
    nbad = int((codes != exp["w_codes"]).sum())
    assert nbad == 0, f"weight codes differ in {nbad} bytes"
    assert np.array_equal(scales, exp["w_scales"]), "weight scales differ"
    return dict(inv_lambda=inv, L1=L1, L2t=L2t, w_codes=codes, w_scales=scales, bias=bias)


# ---------------------------------------------------------------------------
# S1: activation quantisation
# ---------------------------------------------------------------------------

KERNELS = pytest.mark.parametrize("ws", [False, True], ids=["act16", "act128"])


@KERNELS
@pytest.mark.parametrize("M,K,r", [(256, 512, 32), (1, 256, 16), (17, 768, 32), (129, 512, 64),
                                   (300, 1024, 8), (64, 256, 0), (200, 512, 48), (1000, 3072, 32)])
def test_act_quant_parity(M, K, r, ws):
    _act_parity_case(M, K, r, ws)


@KERNELS
@pytest.mark.parametrize("ks", [1, 2, 3, 4, 6, 8])
@pytest.mark.parametrize("r", [32, 64, 0])
def test_act_quant_parity_k_split(ks, r, ws):
    """K split forced to ks: clusters of ks CTAs sharing each 16-row block
    (svdq_quantize_act), or ks CTAs per 128-row block whose float32 partials of
    D the last one adds (the forward's kernel, through svdq_quantize_act_ws)."""
    with svdq.override(svdq.SVDQ_OVERRIDE_ACT_KSPLIT, ks):
        _act_parity_case(40 if not ws else 300, 3072, r, ws)


def _act_parity_case(M, K, r, ws=False):
    X, W, _, lam = _inputs(M, K, max(128, r), seed=M * 7 + K + r)
    inv = ref.inv_lambda_of(lam)
    rng = np.random.default_rng(5)
    L1 = gen.to_bf16_bits(rng.standard_normal((K, r)) * 0.3) if r else None
    codes, scales, full, d = _run_act(X, inv, L1, ws=ws)
    o = ref.quantize_act(X, inv, L1)
    nbad = int((codes != o["x_codes"]).sum())
    assert nbad == 0, f"{nbad} code bytes differ"
    assert np.array_equal(scales, o["x_scales"])
    assert np.all(full[M:] == 0), "padding rows of the scale tiles must be zero"
    if r:
        check_d(d, o["D"], o["D_abs"])


@KERNELS
def test_act_quant_rounding_cases(ws):
    """Exact ties, scale ties, saturation, zero and negative-zero blocks (lambda = 1)."""
    K = 256
    ties = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -0.0]
    rows = []
    for k in range(-6, 7, 2):
        rows.append([v * 2.0 ** k for v in ties] * (K // 16))
    # scale ties: amax/6 = 1.0625 (between E4M3 1.0 and 1.125) and 1.1875
    rows.append(([6.375] + [0.5] * 15) * (K // 16))
    rows.append(([7.125] + [-0.3] * 15) * (K // 16))
    # saturating scale (amax/6 > 448) and saturating codes
    rows.append(([3000.0] + [-2990.0] + [1.0] * 14) * (K // 16))
    # tiny blocks: scale 0, codes keep the sign
    rows.append(([1e-3, -1e-3] * 8) * (K // 16))
    rows.append([0.0] * K)
    # values just off the E2M1 thresholds
    rows.append(([6.0, 0.2501, 0.7499, 1.2501, 1.7499, 2.5001, 3.4999, 5.0001] * 2) * (K // 16))
    X = gen.to_bf16_bits(np.array(rows, dtype=np.float64))
    inv = np.ones(K, np.float32)
    codes, scales, _, _ = _run_act(X, inv, _any_l1(K) if ws else None, ws=ws)
    o = ref.quantize_act(X, inv, None)
    assert np.array_equal(scales, o["x_scales"])
    assert np.array_equal(codes, o["x_codes"]), np.argwhere(codes != o["x_codes"])[:8]


@KERNELS
def test_act_quant_random_lambda_sweep(ws):
    """Many distinct float32 quotients: X and lambda random over wide ranges."""
    rng = np.random.default_rng(77)
    M, K = 512, 2048
    x = rng.standard_normal((M, K)) * np.exp(rng.uniform(-6, 6, (M, 1)))
    X = gen.to_bf16_bits(x)
    lam = np.exp(rng.uniform(-3, 3, K)).astype(np.float32)
    inv = ref.inv_lambda_of(lam)
    codes, scales, _, _ = _run_act(X, inv, _any_l1(K) if ws else None, ws=ws)
    o = ref.quantize_act(X, inv, None)
    assert np.array_equal(scales, o["x_scales"])
    assert int((codes != o["x_codes"]).sum()) == 0


def _any_l1(K, r=16):
    """Some L1 (codes and scales do not depend on it; the forward's kernel needs r > 0)."""
    return gen.to_bf16_bits(np.random.default_rng(3).standard_normal((K, r)) * 0.3)


# ---------------------------------------------------------------------------
# S0: weight preparation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K,r,with_bias", [(512, 512, 32, True), (256, 1024, 16, False),
                                             (1024, 256, 64, True), (384, 768, 0, True),
                                             (128, 256, 8, False)])
def test_prepare_parity(N, K, r, with_bias):
    _, W, B, lam = _inputs(64, K, N, seed=N + K + r)
    bias = B if with_bias else None
    lin, exp = _prepare(W, lam, bias, r)
    _oracle_prep_from_export(W, lam, bias, exp, r)
    if r:
        L1o, L2o, sig = ref.svd_split(ref.smooth_weight(W, lam), r)
        po = ref.bf16_to_f64(L1o) @ ref.bf16_to_f64(L2o)
        pg = ref.bf16_to_f64(exp["L1"]) @ ref.bf16_to_f64(exp["L2t"]).T
        rel = np.linalg.norm(pg - po) / np.linalg.norm(po)
        assert rel <= 1e-2, rel
        # column norms of L1 are the singular values
        cn = np.linalg.norm(ref.bf16_to_f64(exp["L1"]), axis=0)
        assert np.allclose(cn, sig[:r], rtol=1e-2)
        # sign convention
        L1g = ref.bf16_to_f64(exp["L1"])
        for j in range(r):
            assert L1g[np.argmax(np.abs(L1g[:, j])), j] > 0


# ---------------------------------------------------------------------------
# S2 + S3: GEMM with fused low-rank branch and bias
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("BN", [0, 128], ids=["auto", "bn128"])
@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 32), (1, 256, 128, 16), (129, 768, 384, 32),
                                     (300, 1024, 256, 0), (64, 512, 1024, 64), (513, 256, 640, 8),
                                     (700, 1280, 768, 48), (1500, 512, 2048, 32)])
def test_gemm_parity(M, K, N, r, BN):
    """svdq_gemm on oracle-produced activation codes: isolates the tensor-core GEMM
    (128 x 256 or 128 x 128 tiles)."""
    with svdq.override(svdq.SVDQ_OVERRIDE_GEMM_BN, BN):
        _gemm_parity_case(M, K, N, r)


def _gemm_parity_case(M, K, N, r):
    t = torch()
    X, W, B, lam = _inputs(M, K, N, seed=3 * M + K + N + r)
    lin, exp = _prepare(W, lam, B, r)
    prep = _oracle_prep_from_export(W, lam, B, exp, r)
    o = ref.linear_forward(X, prep)
    codes = dev_u8(o["x_codes"])
    native = np.zeros(svdq.svdq_act_scales_bytes(M, K), np.uint8)
    logical = np.ascontiguousarray(o["x_scales"])       # kept alive across the call
    svdq.svdq_scales_to_native(logical.ctypes.data, M, K, native.ctypes.data)
    sc = dev_u8(native)
    D = dev_u16(o["D"]) if r else None
    Y = t.empty((M, N), dtype=t.int16, device="cuda")
    svdq.svdq_gemm(codes.data_ptr(), sc.data_ptr(), D.data_ptr() if r else 0, M, lin.w,
                   Y.data_ptr(), stream())
    t.cuda.synchronize()
    check_y(to_np_u16(Y), o["Y64"], "gemm")


@pytest.mark.parametrize("BN", [128, 256])
def test_gemm_output_16_byte_aligned(BN):
    """Y only 16-byte aligned (the interface's minimum): the epilogue's rows go
    out as two 16-byte stores; rows past M (ragged tail) are never written."""
    with svdq.override(svdq.SVDQ_OVERRIDE_GEMM_BN, BN):
        _gemm_16_byte_case()


def _gemm_16_byte_case():
    t = torch()
    M, K, N, r = 200, 512, 512, 32
    X, W, B, lam = _inputs(M, K, N, seed=77)
    lin, exp = _prepare(W, lam, B, r)
    prep = _oracle_prep_from_export(W, lam, B, exp, r)
    o = ref.linear_forward(X, prep)
    codes = dev_u8(o["x_codes"])
    native = np.zeros(svdq.svdq_act_scales_bytes(M, K), np.uint8)
    logical = np.ascontiguousarray(o["x_scales"])       # kept alive across the call
    svdq.svdq_scales_to_native(logical.ctypes.data, M, K, native.ctypes.data)
    sc = dev_u8(native)
    D = dev_u16(o["D"])
    guard = 0x5A5A
    buf = t.full((M * N + 64,), guard, dtype=t.int16, device="cuda")
    Y = buf[8:8 + M * N]                          # 16 bytes past a 256-byte boundary
    assert Y.data_ptr() % 32 == 16
    svdq.svdq_gemm(codes.data_ptr(), sc.data_ptr(), D.data_ptr(), M, lin.w, Y.data_ptr(), stream())
    t.cuda.synchronize()
    check_y(to_np_u16(Y.view(M, N)), o["Y64"], "gemm, 16-byte aligned Y")
    rest = to_np_u16(buf)
    assert np.all(rest[:8] == guard) and np.all(rest[8 + M * N:] == guard)


# ---------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N,r,with_bias", [(256, 512, 512, 32, True), (1, 256, 256, 32, True),
                                               (129, 1024, 384, 16, False), (777, 512, 1280, 64, True),
                                               (40, 768, 128, 0, False), (2000, 768, 2304, 32, True)])
def test_forward_parity(M, K, N, r, with_bias):
    t = torch()
    X, W, B, lam = _inputs(M, K, N, seed=11 * M + K + N + r)
    bias = B if with_bias else None
    lin, exp = _prepare(W, lam, bias, r)
    prep = _oracle_prep_from_export(W, lam, bias, exp, r)
    Y = lin.forward(dev_u16(X).view(t.bfloat16))
    t.cuda.synchronize()
    o = ref.linear_forward(X, prep)
    yd = y_with_d(o["Y64"], o["D"], gpu_d(lin, dev_u16(X), M), exp["L2t"]) if r else None
    check_y(to_np_u16(Y.view(t.int16)), o["Y64"], "forward", y_given_gpu_d=yd)


@pytest.mark.parametrize("M,K,N,r", [(256, 512, 512, 32), (129, 1024, 384, 16), (777, 3072, 1280, 64),
                                     (3000, 1536, 256, 32), (1, 256, 256, 8)])
def test_forward_parity_tensor_core_activation_kernel(M, K, N, r):
    """The whole layer with the 128-row activation kernel forced (D on the tensor
    cores, K split with float32 partials), at the strict bar."""
    t = torch()
    X, W, B, lam = _inputs(M, K, N, seed=13 * M + K + N + r)
    lin, exp = _prepare(W, lam, B, r)
    prep = _oracle_prep_from_export(W, lam, B, exp, r)
    with svdq.override(svdq.SVDQ_OVERRIDE_ACT_KERNEL, 2):
        Y = lin.forward(dev_u16(X).view(t.bfloat16))
        t.cuda.synchronize()
        Dg = gpu_d(lin, dev_u16(X), M)
    o = ref.linear_forward(X, prep)
    check_d(Dg, o["D"], o["D_abs"])
    yd = y_with_d(o["Y64"], o["D"], Dg, exp["L2t"])
    check_y(to_np_u16(Y.view(t.int16)), o["Y64"], "forward (128-row act)", y_given_gpu_d=yd)
    assert svdq.svdq_get_device_status(stream()) == 0


def test_forward_small_workload_end_to_end():
    """The 256 x 512 x 512 (r = 32) workload: against the oracle on the exported
    weight (the gate) and, loosely, against the oracle's own end-to-end run."""
    t = torch()
    spec = gen.workload("small")
    d = gen.make_linear(spec)
    lin, exp = _prepare(d["W"], d["lam"], d["bias"], spec.r)
    prep = _oracle_prep_from_export(d["W"], d["lam"], d["bias"], exp, spec.r)
    Y = to_np_u16(lin.forward(dev_u16(d["X"]).view(t.bfloat16)).view(t.int16))
    o = ref.linear_forward(d["X"], prep)
    yd = y_with_d(o["Y64"], o["D"], gpu_d(lin, dev_u16(d["X"]), spec.M), exp["L2t"])
    check_y(Y, o["Y64"], "small", y_given_gpu_d=yd)
    # the loose cross-check: the oracle end to end with its own SVD (LAPACK's
    # factors instead of the library's), within 2e-2 rms
    own = ref.linear_forward(d["X"], ref.prepare_weight(d["W"], d["lam"], d["bias"], spec.r))["Y64"]
    rms = np.sqrt(np.mean(own ** 2))
    dev = float(np.max(np.abs(ref.bf16_to_f64(Y) - own)))
    print(f"small, oracle's own SVD: max |dY| / rms = {dev / rms:.3e} (bar 2e-2)")
    assert dev <= 2e-2 * rms


@pytest.mark.parametrize("M", [200, 2600])
def test_forward_host_buffers_match_device_path(M):
    """Host-buffer forward; M = 2600 takes the pipelined path (chunks of 1024
    rows, copies back on a second stream), and only the caller's stream is
    synchronised before Y is read."""
    t = torch()
    K, N, r = 512, 384, 32
    X, W, B, lam = _inputs(M, K, N, seed=91)
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


def test_forward_host_buffers_concurrent_callers():
    """Two host threads drive the pipelined host-buffer path at the same time on
    their own streams (the copy-out stream and events are shared per device):
    each result must equal its device-path result."""
    import threading
    t = torch()
    M, K, N, r = 2600, 512, 384, 32
    runs = []
    for seed in (92, 93):
        X, W, B, lam = _inputs(M, K, N, seed=seed)
        lin, _ = _prepare(W, lam, B, r)
        Yd = to_np_u16(lin.forward(dev_u16(X).view(t.bfloat16)).view(t.int16))
        nb = lin.workspace_bytes(M)
        runs.append(dict(lin=lin, Yd=Yd, nb=nb, ws=empty_u8(nb), st=t.cuda.Stream(),
                         Xh=t.from_numpy(X.view(np.int16).copy()).pin_memory(),
                         Yh=t.empty((M, N), dtype=t.int16).pin_memory(),
                         Xdev=t.empty((M, K), dtype=t.int16, device="cuda"),
                         Ydev=t.empty((M, N), dtype=t.int16, device="cuda")))
    t.cuda.synchronize()
    errors = []

    def drive(rr):
        try:
            for _ in range(3):
                svdq.svdq_linear_forward_host(rr["Xh"].data_ptr(), M, rr["lin"].w, rr["Yh"].data_ptr(),
                                              rr["Xdev"].data_ptr(), rr["Ydev"].data_ptr(),
                                              rr["ws"].data_ptr(), rr["nb"], int(rr["st"].cuda_stream))
        except Exception as e:   # reported on the main thread
            errors.append(e)

    threads = [threading.Thread(target=drive, args=(rr,)) for rr in runs]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors, errors
    for rr in runs:
        rr["st"].synchronize()
        assert np.array_equal(rr["Yh"].numpy().view(np.uint16), rr["Yd"])


def test_empty_and_invalid_calls():
    t = torch()
    M, K, N, r = 64, 256, 128, 16
    X, W, B, lam = _inputs(M, K, N, seed=5)
    lin, _ = _prepare(W, lam, B, r)
    Y = t.full((M, N), 7, dtype=t.int16, device="cuda")
    ws = empty_u8(lin.workspace_bytes(M))
    svdq.svdq_linear_forward(dev_u16(X).data_ptr(), 0, lin.w, Y.data_ptr(), ws.data_ptr(), 0, stream())
    t.cuda.synchronize()
    assert int((Y != 7).sum()) == 0, "M = 0 must not touch Y"
    with pytest.raises(svdq.SvdqError, match="WORKSPACE_TOO_SMALL"):
        svdq.svdq_linear_forward(dev_u16(X).data_ptr(), M, lin.w, Y.data_ptr(), ws.data_ptr(), 16,
                                 stream())
    with pytest.raises(svdq.SvdqError, match="MISALIGNED"):
        svdq.svdq_linear_forward(dev_u16(X).data_ptr() + 2, M, lin.w, Y.data_ptr(), ws.data_ptr(),
                                 lin.workspace_bytes(M), stream())


def test_quantiser_quotient_exhaustive():
    """The activation kernel's division-free quotient equals IEEE division, and
    its E2M1 codes (sign kept, ties to even) equal the format's definition, for
    every E4M3 scale and every float32 significand in five binades."""
    q_bad, c_bad, q_sub = svdq.svdq_selftest_quotient()
    # subnormal quotients may differ (q_sub), but their codes are checked too
    assert (q_bad, c_bad) == (0, 0), (q_bad, c_bad, q_sub)


def test_device_conversions_exhaustive():
    """The hardware E4M3, E2M1 and bf16 conversions the kernels round with agree
    with the formats' definitions on every non-negative finite float32 (the
    oracle's table-driven conversions are pinned to the same definitions by
    the CPU tests)."""
    assert svdq.svdq_selftest_conversions() == (0, 0, 0)


def test_device_status_clean():
    torch().cuda.synchronize()
    assert svdq.svdq_get_device_status(stream()) == 0
