"""Pins of the oracle's smoothing, rank-r split and residual.

References independent of the oracle's own formulas: f64 algebra identities
(smoothing followed by its inverse), the full-rank reconstruction (residual
exactly zero), the Eckart-Young theorem, orthonormality of singular vectors,
and the quality sanity of the method (error falls with the rank and with
smoothing).
"""
import numpy as np
import pytest

from oracle import svdq_ref as ref
from workloads import gen


def _inputs(M, K, N, seed, spike=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    x[:, rng.choice(K, 3, replace=False)] *= 40
    w = rng.standard_normal((N, K)) * 0.02
    w[:, rng.choice(K, 2, replace=False)] *= 10
    if spike:
        u, _ = np.linalg.qr(rng.standard_normal((N, 4)))
        v, _ = np.linalg.qr(rng.standard_normal((K, 4)))
        w += 5 * u @ v.T
    X, W = gen.to_bf16_bits(x), gen.to_bf16_bits(w)
    return X, W, gen.calibrate_lambda(X, W)


def test_smoothing_identity_f64():
    """X diag(1/lambda) . (W diag(lambda))^T == X W^T in float64 (to rounding)."""
    X, W, lam = _inputs(32, 96, 40, 1)
    inv64 = 1.0 / lam.astype(np.float64)
    xh = ref.smooth_act(X, inv64, dtype=np.float64)
    wh = ref.smooth_weight(W, lam.astype(np.float64), dtype=np.float64)
    y = ref.bf16_to_f64(X) @ ref.bf16_to_f64(W).T
    assert np.max(np.abs(xh @ wh.T - y)) <= 1e-13 * np.abs(y).max()
    # the smoothing really acts on input channels (columns): a channel with lambda = 2
    lam2 = np.ones(96, np.float32)
    lam2[5] = 2.0
    xh2 = ref.smooth_act(X, ref.inv_lambda_of(lam2))
    assert np.array_equal(xh2[:, 5], (ref.bf16_to_f64(X)[:, 5] / 2).astype(np.float32))
    assert np.array_equal(np.delete(xh2, 5, 1), np.delete(ref.bf16_to_f64(X), 5, 1).astype(np.float32))
    wh2 = ref.smooth_weight(W, lam2)
    assert np.array_equal(wh2[:, 5], (ref.bf16_to_f64(W)[:, 5] * 2).astype(np.float32))


@pytest.mark.parametrize("K,N", [(48, 32), (32, 80), (64, 64)])
def test_full_rank_reconstruction(K, N):
    """r = min(K, N), f64 factors: residual is zero and the low-rank branch is X W^T."""
    X, W, lam = _inputs(16, K, N, 2)
    wh = ref.smooth_weight(W, lam.astype(np.float64), dtype=np.float64)
    r = min(K, N)
    L1, L2, sig = ref.svd_split(wh, r, round_bf16=False)
    R = ref.residual(wh, L1, L2)
    assert np.max(np.abs(R)) <= 1e-12 * np.abs(wh).max()
    xh = ref.smooth_act(X, 1.0 / lam.astype(np.float64), dtype=np.float64)
    y_low = (xh @ L1) @ L2
    y = ref.bf16_to_f64(X) @ ref.bf16_to_f64(W).T
    assert np.max(np.abs(y_low - y)) <= 1e-10 * np.abs(y).max()


@pytest.mark.parametrize("r", [1, 4, 8, 17])
def test_eckart_young_and_orthonormality(r):
    _, W, lam = _inputs(8, 64, 48, 3, spike=True)
    wh = ref.smooth_weight(W, lam)
    L1, L2, sig = ref.svd_split(wh, r, round_bf16=False)
    a = wh.astype(np.float64).T
    err = np.linalg.norm(a - L1 @ L2, "fro") ** 2
    assert abs(err - np.sum(sig[r:] ** 2)) <= 1e-10 * np.sum(sig ** 2)
    # L2 rows orthonormal; L1 columns orthogonal with norms sigma
    assert np.allclose(L2 @ L2.T, np.eye(r), atol=1e-12)
    g = L1.T @ L1
    assert np.allclose(g, np.diag(sig[:r] ** 2), atol=1e-10 * sig[0] ** 2)
    # sign convention: largest-|.| entry of each u_i is positive
    for i in range(r):
        col = L1[:, i]
        assert col[np.argmax(np.abs(col))] > 0
    # K x r and r x N, per the reading What^T = L1 L2 (+ residual)
    assert L1.shape == (64, r) and L2.shape == (r, 48)


def test_residual_absorbs_bf16_rounding():
    _, W, lam = _inputs(8, 64, 32, 4)
    wh = ref.smooth_weight(W, lam)
    L1b, L2b, _ = ref.svd_split(wh, 8)
    R, _, _ = ref.residual_quantize(wh, L1b, L2b)
    recon = R.astype(np.float64) + (ref.bf16_to_f64(L1b) @ ref.bf16_to_f64(L2b)).T
    # R is the float32 rounding of the exact residual: reconstruction error <= half ulp of R
    ulp = np.spacing(np.abs(R).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(recon - wh.astype(np.float64)) <= ulp / 2 + 1e-300)


def test_quality_sanity_error_falls_with_rank_and_smoothing():
    """Not a parity pin: the method must do its job on DiT-like outliers."""
    rng = np.random.default_rng(5)
    M, K, N = 128, 256, 384
    x = rng.standard_normal((M, K))
    x[:, rng.choice(K, 4, replace=False)] *= 50
    w = rng.standard_normal((N, K)) * 0.02
    u, _ = np.linalg.qr(rng.standard_normal((N, 8)))
    v, _ = np.linalg.qr(rng.standard_normal((K, 8)))
    w += 5 * u @ v.T / np.sqrt(K / 256)
    X, W = gen.to_bf16_bits(x), gen.to_bf16_bits(w)
    y = ref.bf16_to_f64(X) @ ref.bf16_to_f64(W).T
    lam = gen.calibrate_lambda(X, W)

    def err(lam_, r):
        prep = ref.prepare_weight(W, lam_, None, r)
        yq = ref.linear_forward(X, prep)["Y64"]
        return np.linalg.norm(yq - y) / np.linalg.norm(y)

    e0, e8, e32 = err(lam, 0), err(lam, 8), err(lam, 32)
    e32_nosmooth = err(np.ones(K, np.float32), 32)
    assert e32 < e8 < e0
    assert e32 < e32_nosmooth
