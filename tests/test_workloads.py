"""The seeded input recipe (workloads/gen.py) against the statement of it:
shapes, determinism, outlier channels, the GELU-shaped down-projection input,
the rank-8 spike of the QKV weight, the bias scale and the lambda recipe."""
import numpy as np
import pytest

from workloads import gen

SHAPES = {
    "small": (256, 512, 512, 32), "qkv": (4608, 3072, 9216, 32), "mlp_up": (4608, 3072, 12288, 32),
    "mlp_down": (4608, 12288, 3072, 32), "small_m": (16, 3072, 18432, 32),
    "block_b1_qkv": (4608, 3072, 9216, 32), "block_b1_out": (4608, 3072, 3072, 32),
    "block_b1_up": (4608, 3072, 12288, 32), "block_b1_down": (4608, 12288, 3072, 32),
    "block_b4_qkv": (18432, 3072, 9216, 32), "block_b4_down": (18432, 12288, 3072, 32),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_shapes(name):
    s = gen.workload(name)
    assert (s.M, s.K, s.N, s.r) == SHAPES[name]
    assert s.flops == 2 * s.M * s.N * s.K


def _outlier_columns(X, threshold):
    return int((np.abs(gen.bf16_bits_to_f32(X)).max(axis=0) > threshold).sum())


def test_small_recipe_and_determinism():
    s = gen.workload("small")
    a, b = gen.make_linear(s), gen.make_linear(s)
    for k in ("X", "W", "bias", "lam"):
        assert np.array_equal(a[k], b[k])
    assert a["X"].dtype == np.uint16 and a["X"].shape == (256, 512)
    assert _outlier_columns(a["X"], 20.0) == 4                   # 4 channels x40
    w = np.abs(gen.bf16_bits_to_f32(a["W"])).max(axis=0)
    assert int((w > 0.12).sum()) == 2                             # 2 weight columns x10
    bias = gen.bf16_bits_to_f32(a["bias"]).astype(np.float64)
    assert 0.006 < bias.std() < 0.014


def test_lambda_recipe():
    d = gen.make_linear(gen.workload("small"))
    xm = np.abs(gen.bf16_bits_to_f32(d["X"]).astype(np.float64)).max(axis=0)
    wm = np.abs(gen.bf16_bits_to_f32(d["W"]).astype(np.float64)).max(axis=0)
    assert np.array_equal(d["lam"], np.sqrt(xm / wm).astype(np.float32))
    z = gen.calibrate_lambda(np.zeros((4, 8), np.uint16), gen.to_bf16_bits(np.ones((3, 8))))
    assert np.all(z == 1.0)                                       # a zero channel keeps lambda = 1


def test_qkv_outliers_and_rank8_spike():
    from scipy.sparse.linalg import svds
    d = gen.make_linear(gen.workload("qkv"))
    assert _outlier_columns(d["X"], 25.0) == 31                  # round(1% of 3072) channels x50
    W = gen.bf16_bits_to_f32(d["W"]).astype(np.float64)
    sv = np.sort(svds(W, k=10, return_singular_vectors=False))[::-1]
    assert np.all((sv[:8] > 4.5) & (sv[:8] < 6.5)), sv           # 8 directions of singular value 5
    assert sv[8] < 3.6, sv                                        # then the N(0, 0.02) bulk edge


def test_down_projection_input_is_gelu_shaped():
    d = gen.make_linear(gen.workload("mlp_down"), M=64)
    x = gen.bf16_bits_to_f32(d["X"]).astype(np.float64)
    big = np.abs(x).max(axis=0) > 15.0
    assert int(big.sum()) == 61                                   # round(0.5% of 12288) channels x30
    assert x[:, ~big].min() >= -0.171                             # GELU-tanh's minimum is about -0.170
