"""Pins of the oracle's calibration step (smoothing factors from statistics)."""
import numpy as np
import pytest

from oracle import svdq_ref as ref
from workloads import gen


def _mats(seed=0, M=64, N=48, K=32):
    rng = np.random.default_rng(seed)
    X = gen.to_bf16_bits(rng.standard_normal((M, K)) * rng.uniform(0.1, 30.0, K))
    W = gen.to_bf16_bits(rng.standard_normal((N, K)) * 0.02)
    return X, W


def test_column_absmax_is_exact_maximum():
    X, _ = _mats(1)
    want = np.array([max(abs(float(v)) for v in ref.bf16_to_f64(X[:, k])) for k in range(X.shape[1])])
    assert np.array_equal(ref.column_absmax(X).astype(np.float64), want)


def test_balance_at_half_migration():
    """alpha = 0.5: after smoothing, each channel's activation and weight maxima
    coincide (x / lambda = w * lambda = sqrt(x w)), up to float32 rounding."""
    X, W = _mats(2)
    xm = ref.column_absmax(X).astype(np.float64)
    lam = ref.calibrate_lambda(ref.column_absmax(X), W, 0.5).astype(np.float64)
    wm = ref.column_absmax(W).astype(np.float64)
    assert np.allclose(xm / lam, wm * lam, rtol=2.0 ** -22)


@pytest.mark.parametrize("alpha,j", [(0.5, 2), (0.25, 4), (0.75, 4)])
def test_power_of_two_homogeneity(alpha, j):
    """Scaling column k of X by 2^j scales lambda_k by 2^(j alpha), and scaling
    column k of W by 2^j scales it by 2^(-j (1 - alpha)); exact when those
    exponents are integers."""
    X, W = _mats(3)
    xm = ref.column_absmax(X)
    lam = ref.calibrate_lambda(xm, W, alpha)
    lam_x = ref.calibrate_lambda(xm * np.float32(2.0 ** j), W, alpha)
    assert np.array_equal(lam_x, lam * np.float32(2.0 ** (j * alpha)))
    W2 = gen.to_bf16_bits(ref.bf16_to_f64(W) * 2.0 ** j)
    lam_w = ref.calibrate_lambda(xm, W2, alpha)
    assert np.array_equal(lam_w, (lam.astype(np.float64) * 2.0 ** (-j * (1 - alpha))).astype(np.float32))


def test_migration_extremes_and_zero_columns():
    X, W = _mats(4)
    xm = ref.column_absmax(X)
    wm = ref.column_absmax(W)
    assert np.array_equal(ref.calibrate_lambda(xm, W, 1.0), xm)                      # all into W
    assert np.allclose(ref.calibrate_lambda(xm, W, 0.0), 1.0 / wm.astype(np.float64), rtol=2.0 ** -23)
    X[:, 3] = 0
    W[:, 5] = 0
    lam = ref.calibrate_lambda(ref.column_absmax(X), W, 0.5)
    assert lam[3] == 1.0 and lam[5] == 1.0


def test_half_migration_matches_input_recipe():
    """The workloads' lambda (gen.calibrate_lambda, used by every config) is the
    alpha = 0.5 calibration on the layer's own input."""
    X, W = _mats(5)
    assert np.array_equal(ref.calibrate_lambda(ref.column_absmax(X), W, 0.5), gen.calibrate_lambda(X, W))
