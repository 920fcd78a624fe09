"""Offline tooling on the GPU: calibration statistics and smoothing factors
against the oracle, and the checkpoint path (export -> import, save -> load)
reproducing the layer bit for bit."""
import numpy as np
import pytest

from oracle import svdq_ref as ref
from workloads import gen

from gpu_util import dev_f32, dev_u16, stream, to_np_u16, torch

pytestmark = pytest.mark.gpu

svdq = pytest.importorskip("w4a4_rank_corrected_act_b200")


def _calib_inputs(seed, K=384, N=256):
    rng = np.random.default_rng(seed)
    scales = rng.uniform(0.05, 40.0, K)
    batches = [gen.to_bf16_bits(rng.standard_normal((m, K)) * scales) for m in (37, 200, 1)]
    batches[1][:, 7] = 0                      # a channel that never fires in that batch
    for b in batches:
        b[:, 11] = 0                          # a channel that never fires at all
    W = gen.to_bf16_bits(rng.standard_normal((N, K)) * 0.02)
    W[:, 13] = 0                              # an input channel the weight ignores
    return batches, W


def test_calib_absmax_running_maximum_is_exact():
    t = torch()
    batches, _ = _calib_inputs(1)
    K = batches[0].shape[1]
    colmax = t.zeros(K, dtype=t.float32, device="cuda")
    for b in batches:
        svdq.svdq_calib_absmax(dev_u16(b).data_ptr(), b.shape[0], K, colmax.data_ptr(), stream())
    t.cuda.synchronize()
    want = ref.column_absmax(np.concatenate(batches, axis=0))
    assert np.array_equal(colmax.cpu().numpy().view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("alpha", [0.5, 0.25, 0.75, 1.0, 0.0])
def test_calibrate_lambda_matches_oracle(alpha):
    t = torch()
    batches, W = _calib_inputs(2)
    X = [dev_u16(b) for b in batches]
    lam = svdq.calibrate_lambda(dev_u16(W).view(t.bfloat16), [x.view(t.bfloat16) for x in X], alpha)
    t.cuda.synchronize()
    got = lam.cpu().numpy()
    want = ref.calibrate_lambda(ref.column_absmax(np.concatenate(batches, axis=0)), W, alpha)
    if alpha == 0.5:
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    else:
        # float64 pow of the device and of the host may differ in the last bit
        # before the float32 rounding: at most one float32 step apart
        diff = np.abs(got.view(np.int32).astype(np.int64) - want.view(np.int32).astype(np.int64))
        assert diff.max() <= 1
    assert got[11] == 1.0 and got[13] == 1.0


def test_calibrate_rejects_bad_alpha():
    t = torch()
    x = t.zeros(64, dtype=t.float32, device="cuda")
    W = t.zeros((128, 64), dtype=t.int16, device="cuda")
    lam = t.empty(64, dtype=t.float32, device="cuda")
    with pytest.raises(svdq.SvdqError, match="INVALID_ARG"):
        svdq.svdq_calibrate_lambda(x.data_ptr(), W.data_ptr(), 128, 64, 1.5, lam.data_ptr(), stream())


def _layer(seed, M=130, K=512, N=384, r=32, bias=True):
    spec = gen.LinearSpec("tool", M, K, N, r, seed)
    d = gen.make_linear(spec)
    lin = svdq.SvdqLinear(dev_u16(d["W"]), dev_f32(d["lam"]), dev_u16(d["bias"]) if bias else None, r=r)
    torch().cuda.synchronize()
    return lin, d


@pytest.mark.parametrize("r,bias", [(32, True), (0, False), (64, True)])
def test_export_import_reproduces_the_layer(r, bias):
    t = torch()
    lin, d = _layer(3 + r, r=r, bias=bias)
    exp = lin.export()
    twin = svdq.SvdqLinear.from_export(exp, bias=lin.bias_host())
    X = dev_u16(d["X"]).view(t.bfloat16)
    y0 = to_np_u16(lin.forward(X).view(t.int16))
    y1 = to_np_u16(twin.forward(X).view(t.int16))
    t.cuda.synchronize()
    assert np.array_equal(y0, y1)
    exp2 = twin.export()
    for k in exp:
        assert np.array_equal(exp[k], exp2[k]), k


def test_save_load_file_round_trip(tmp_path):
    t = torch()
    lin, d = _layer(9)
    path = tmp_path / "layer.npz"
    lin.save(path)
    back = svdq.SvdqLinear.load(path)
    X = dev_u16(d["X"]).view(t.bfloat16)
    assert np.array_equal(to_np_u16(lin.forward(X).view(t.int16)), to_np_u16(back.forward(X).view(t.int16)))


def test_import_checks_the_bias_field():
    lin, _ = _layer(11)
    exp = lin.export()
    # a weight bound with a bias field needs one
    w = svdq.SvdqLinear.__new__(svdq.SvdqLinear)
    w._bind(lin.N, lin.K, lin.r, True, "cuda")
    with pytest.raises(svdq.SvdqError, match="INVALID_ARG"):
        svdq.svdq_weight_import(w.w, exp["w_codes"].ctypes.data, exp["w_scales"].ctypes.data,
                                exp["L1"].ctypes.data, exp["L2t"].ctypes.data,
                                exp["inv_lambda"].ctypes.data, 0, stream())
