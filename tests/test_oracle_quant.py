"""Pins of the oracle's block quantiser, packing and whole forward.

Independent references: hand-derived blocks (tests/golden/nvfp4_blocks.txt),
exact round trips of representable blocks, power-of-two scaling invariance,
and the brute-force twin (explicit loops, closed-form conversions).
"""
import os

import numpy as np
import pytest

from oracle import brute
from oracle import svdq_ref as ref
from workloads import gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_blocks():
    out = []
    with open(os.path.join(GOLDEN, "nvfp4_blocks.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            name, vals, sc, packed = [p.strip() for p in line.split("|")]
            out.append((name, [float(v) for v in vals.split()], int(sc, 16),
                        [int(b, 16) for b in packed.split()]))
    return out


@pytest.mark.parametrize("name,vals,scale,packed", _golden_blocks())
def test_golden_blocks(name, vals, scale, packed):
    v = np.array([vals], dtype=np.float32)
    codes, scales = ref.quantize_blocks(v)
    assert int(scales[0, 0]) == scale
    assert list(ref.pack_nibbles(codes)[0]) == packed


def test_packing_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    assert list(ref.pack_nibbles(codes)[0]) == [0x21, 0x43, 0x0F]
    assert np.array_equal(ref.unpack_nibbles(ref.pack_nibbles(codes)), codes)


def test_representable_block_roundtrip():
    """A block s*{E2M1 values} with s an E4M3 value and max = 6s comes back exactly."""
    rng = np.random.default_rng(21)
    for _ in range(200):
        s_code = int(rng.integers(8, 0x70))          # normal scales, away from saturation
        s = ref.e4m3_decode(np.array([s_code], np.uint8))[0]
        c = rng.integers(0, 16, 16).astype(np.uint8)
        c[int(rng.integers(0, 16))] = 7 | (8 if rng.random() < 0.5 else 0)   # max = 6s
        v = (ref.e2m1_decode(c) * s).astype(np.float32)
        codes, scales = ref.quantize_blocks(v[None, :])
        assert int(scales[0, 0]) == s_code
        # -0 codes may come back as +0 only when the input was +0; compare values
        assert np.array_equal(ref.e2m1_decode(codes[0]) * s, v.astype(np.float64))


def test_power_of_two_scaling_invariance():
    rng = np.random.default_rng(22)
    v = (rng.standard_normal((64, 32)) * 0.3).astype(np.float32)
    c0, s0 = ref.quantize_blocks(v)
    for k in (-3, -1, 1, 2, 4):
        ck, sk = ref.quantize_blocks((v * np.float32(2.0 ** k)).astype(np.float32))
        d0, dk = ref.e4m3_decode(s0), ref.e4m3_decode(sk)
        ok = (d0 >= 2 ** -6) & (d0 * 2.0 ** k >= 2 ** -6) & (d0 * 2.0 ** k <= 448)
        assert np.all(dk[ok] == d0[ok] * 2.0 ** k)
        blk_ok = np.repeat(ok, 16, axis=1)
        assert np.array_equal(ck[blk_ok], c0[blk_ok])


def test_zero_block_and_tiny_block():
    v = np.zeros((1, 16), np.float32)
    v[0, 3] = -0.0
    c, s = ref.quantize_blocks(v)
    assert s[0, 0] == 0 and c[0, 3] == 8 and c[0, 0] == 0
    # amax below half the smallest scale: s = 0, codes keep the sign
    t = np.full((1, 16), 1e-4, np.float32)
    t[0, 1] = -1e-4
    c, s = ref.quantize_blocks(t)
    assert s[0, 0] == 0 and c[0, 0] == 0 and c[0, 1] == 8


def test_dequantize_matches_definition():
    rng = np.random.default_rng(23)
    v = (rng.standard_normal((3, 48))).astype(np.float32)
    c, s = ref.quantize_blocks(v)
    d = ref.dequantize(ref.pack_nibbles(c), s)
    for i in range(3):
        for k in range(48):
            assert d[i, k] == brute.code_value(int(c[i, k])) * brute.e4m3_value(int(s[i, k // 16]))


@pytest.mark.parametrize("M,N,K,r", [(1, 1, 16, 0), (3, 16, 32, 1), (16, 3, 64, 3), (16, 16, 32, 4),
                                     (16, 16, 64, 4), (3, 3, 16, 1), (1, 16, 32, 0)])
def test_brute_force_twin(M, N, K, r):
    rng = np.random.default_rng(1000 + M * 100 + N * 10 + K + r)
    X = gen.random_bf16(rng, (M, K))
    X[:, 0] = gen.to_bf16_bits(gen.bf16_bits_to_f32(X[:, 0]).astype(np.float64) * 30)
    W = gen.random_bf16(rng, (N, K), 0.05)
    bias = gen.random_bf16(rng, (N,), 0.01)
    lam = gen.calibrate_lambda(X, W)
    inv = ref.inv_lambda_of(lam)
    w_hat = ref.smooth_weight(W, lam)
    if r:
        L1, L2, _ = ref.svd_split(w_hat, r)
    else:
        L1 = np.zeros((K, 0), np.uint16)
        L2 = np.zeros((0, N), np.uint16)
    _, wc, ws = ref.residual_quantize(w_hat, L1, L2)
    prep = dict(inv_lambda=inv, L1=L1, L2t=np.ascontiguousarray(L2.T), w_codes=wc,
                w_scales=ws, bias=bias)
    o = ref.linear_forward(X, prep)
    b = brute.forward(X.tolist(), W.tolist(), lam.tolist(), bias.tolist(),
                      L1.tolist(), L2.tolist())
    assert np.array_equal(ref.unpack_nibbles(o["x_codes"]), np.array(b["x_codes"], np.uint8))
    assert np.array_equal(o["x_scales"], np.array(b["x_scales"], np.uint8))
    assert np.array_equal(ref.unpack_nibbles(wc), np.array(b["w_codes"], np.uint8))
    assert np.array_equal(ws, np.array(b["w_scales"], np.uint8))
    if r:
        assert np.array_equal(ref.bf16_to_f64(o["D"]), np.array(b["D"]))
    y_b = np.array(b["Y64"])
    scale = max(np.abs(y_b).max(), 1e-30)
    assert np.max(np.abs(o["Y64"] - y_b)) <= 1e-12 * scale


def test_forward_r0_lambda1_is_plain_nvfp4_gemm():
    """r = 0, lambda = 1: Y = deq(Q(X)) deq(Q(W))^T + b (independent composition)."""
    rng = np.random.default_rng(31)
    M, N, K = 5, 7, 64
    X = gen.random_bf16(rng, (M, K))
    W = gen.random_bf16(rng, (N, K), 0.1)
    bias = gen.random_bf16(rng, (N,), 0.01)
    lam = np.ones(K, np.float32)
    w_hat = ref.smooth_weight(W, lam)
    assert np.array_equal(w_hat, gen.bf16_bits_to_f32(W))
    z1, z2 = np.zeros((K, 0), np.uint16), np.zeros((0, N), np.uint16)
    _, wc, ws = ref.residual_quantize(w_hat, z1, z2)
    prep = dict(inv_lambda=ref.inv_lambda_of(lam), L1=z1, L2t=z2.T, w_codes=wc, w_scales=ws,
                bias=bias)
    y = ref.linear_forward(X, prep)["Y64"]
    cx, sx = ref.quantize_blocks(gen.bf16_bits_to_f32(X))
    cw, sw = ref.quantize_blocks(gen.bf16_bits_to_f32(W))
    # dequantise by explicit per-element loops and an explicit triple loop
    want = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += (brute.code_value(int(cx[m, k])) * brute.e4m3_value(int(sx[m, k // 16])) *
                        brute.code_value(int(cw[n, k])) * brute.e4m3_value(int(sw[n, k // 16])))
            want[m, n] = acc + float(ref.bf16_to_f64(bias[n:n + 1])[0])
    assert np.max(np.abs(y - want)) <= 1e-12 * np.abs(want).max()


def test_y_rounding_is_single_rne_of_f64_sum():
    rng = np.random.default_rng(41)
    M, N, K, r = 4, 8, 32, 2
    X = gen.random_bf16(rng, (M, K))
    W = gen.random_bf16(rng, (N, K), 0.1)
    lam = gen.calibrate_lambda(X, W)
    prep = ref.prepare_weight(W, lam, None, r)
    o = ref.linear_forward(X, prep)
    assert np.array_equal(o["Y"], ref.f64_to_bf16(o["Y64"]))
    assert prep["L1"].shape == (K, r) and prep["L2t"].shape == (N, r)
