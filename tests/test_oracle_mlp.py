"""Pins of the MLP-pair oracle (oracle/mlp_ref.py): the tanh-GELU against its
exact algebraic identity and against the erf GELU (a library routine), and the
whole pair against a scalar-loop composition of the brute-force twin."""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest
from scipy.special import erf

from oracle import brute
from oracle import mlp_ref
from oracle import svdq_ref as ref
from workloads import gen


def test_gelu_tanh_identities():
    x = np.linspace(-8, 8, 4001)
    g = mlp_ref.gelu_tanh_f64(x)
    # y/2 (1 + tanh u) - (-y)/2 (1 + tanh(-u)) = y exactly
    assert np.max(np.abs(g - mlp_ref.gelu_tanh_f64(-x) - x)) <= 1e-14 * 8
    assert mlp_ref.gelu_tanh_f64(np.array([0.0]))[0] == 0.0
    assert mlp_ref.gelu_tanh_f64(np.array([30.0]))[0] == 30.0
    assert abs(mlp_ref.gelu_tanh_f64(np.array([-30.0]))[0]) < 1e-300 + 1e-12


def test_gelu_tanh_close_to_the_erf_gelu():
    x = np.linspace(-6, 6, 12001)
    exact = 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))
    # the tanh form is a published approximation of x Phi(x): a few 1e-4 at most
    assert np.max(np.abs(mlp_ref.gelu_tanh_f64(x) - exact)) < 5e-4
    assert np.min(mlp_ref.gelu_tanh_f64(x)) == pytest.approx(-0.17, abs=0.01)


def _gelu_decimal(y: float) -> float:
    """y/2 (1 + tanh u) in 60-digit decimal arithmetic, tanh from its exponential
    definition: an independent evaluation of the function, exact to far below
    float64 rounding (no cancellation at 60 digits for |u| < 60)."""
    getcontext().prec = 60
    pi = Decimal("3.14159265358979323846264338327950288419716939937510582097494")
    d = Decimal(y)
    u = (Decimal(2) / pi).sqrt() * (d + Decimal("0.044715") * d ** 3)
    e = (2 * u).exp()
    return float(d / 2 * (1 + (e - 1) / (e + 1)))


def _gelu_ref(v: float) -> float:
    return _gelu_decimal(v) if abs(v) < 40 else (v if v > 0 else -0.0)


def test_hidden_is_one_rounding_of_the_gelu():
    rng = np.random.default_rng(1)
    y = gen.to_bf16_bits(rng.standard_normal(2000) * 3)
    h = mlp_ref.mlp_hidden(y)
    for yb, hb in zip(y[:200], h[:200]):
        yv = float(ref.bf16_to_f64(np.array([yb]))[0])
        assert float(ref.bf16_to_f64(np.array([hb]))[0]) == brute.bf16_round(_gelu_ref(yv))


def test_hidden_in_the_negative_tail():
    """Down to y = -12 the tanh-GELU is a tiny, non-zero number (normal bf16 to
    about y = -10, subnormal below): the oracle's H is the single rounding of it
    there too, where 1 + tanh u would cancel in float64."""
    ys = np.concatenate([np.linspace(-12.0, -4.0, 321), [-5.5, -7.8125, -10.0, -10.25]])
    yb = gen.to_bf16_bits(ys)
    h = ref.bf16_to_f64(mlp_ref.mlp_hidden(yb))
    for yv, hv in zip(ref.bf16_to_f64(yb), h):
        want = brute.bf16_round(_gelu_ref(float(yv)))
        assert hv == want, (yv, hv, want)
    assert np.all(h[ref.bf16_to_f64(yb) > -10.0] < 0.0)


def _prep(W, lam, bias, r):
    w_hat = ref.smooth_weight(W, lam)
    if r:
        L1, L2, _ = ref.svd_split(w_hat, r)
    else:
        L1, L2 = np.zeros((W.shape[1], 0), np.uint16), np.zeros((0, W.shape[0]), np.uint16)
    _, wc, ws = ref.residual_quantize(w_hat, L1, L2)
    return dict(inv_lambda=ref.inv_lambda_of(lam), L1=L1, L2=L2, L2t=np.ascontiguousarray(L2.T),
                w_codes=wc, w_scales=ws, bias=bias)


@pytest.mark.parametrize("r", [0, 2])
def test_pair_against_brute_force_composition(r):
    rng = np.random.default_rng(40 + r)
    M, K, F = 3, 32, 48                         # F: hidden width
    X = gen.random_bf16(rng, (M, K))
    W1 = gen.random_bf16(rng, (F, K), 0.2)
    W2 = gen.random_bf16(rng, (K, F), 0.2)
    b1 = gen.random_bf16(rng, (F,), 0.01)
    b2 = gen.random_bf16(rng, (K,), 0.01)
    lam1 = gen.calibrate_lambda(X, W1)
    p1 = _prep(W1, lam1, b1, r)
    lam2 = np.ones(F, np.float32)
    p2 = _prep(W2, lam2, b2, r)
    out = mlp_ref.mlp_pair_forward(X, p1, p2)
    # the brute twin, step by step: up-projection, GELU (math.tanh), down-projection
    up = brute.forward(X.tolist(), W1.tolist(), lam1.tolist(), b1.tolist(), p1["L1"].tolist(),
                       p1["L2"].tolist())
    y_up = [[brute.bf16_round(v) for v in row] for row in up["Y64"]]
    h = [[brute.bf16_round(_gelu_ref(v)) for v in row] for row in y_up]
    assert np.array_equal(ref.bf16_to_f64(out["H"]), np.array(h))
    down = brute.forward(out["H"].tolist(), W2.tolist(), lam2.tolist(), b2.tolist(), p2["L1"].tolist(),
                         p2["L2"].tolist())
    y_b = np.array(down["Y64"])
    assert np.max(np.abs(out["Y64"] - y_b)) <= 1e-12 * max(np.abs(y_b).max(), 1e-30)
