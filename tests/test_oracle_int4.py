"""Pins of the INT4 variant's oracle (oracle/int4_ref.py) against facts fixed
outside it: IEEE binary16 rounding worked by hand, the integer grid of the
format, closed-form round trips, homogeneity, an error bound and the
brute-force twin written with Python scalars and struct-based half rounding.

The pages name INT4 as the pre-Blackwell format of the same layer
(chaosnode.de "Nunchaku Lite", section "Hardware-Support") but print no
detail of it; the format is the reading stated in the oracle's header.
"""
import numpy as np
import pytest

from oracle import brute
from oracle import int4_ref as i4
from oracle import svdq_ref as ref
from workloads import gen


def test_half_rounding_hand_cases():
    cases = [
        (1.0, 0x3C00),
        (1.0 + 2.0 ** -11, 0x3C00),        # tie between 1 and 1 + 2^-10: even mantissa
        (1.0 + 3 * 2.0 ** -11, 0x3C02),    # tie between 1 + 2^-10 and 1 + 2^-9: even
        (65504.0, 0x7BFF),
        (65519.0, 0x7BFF),                 # below the 65520 midpoint
        (70000.0, 0x7BFF),                 # saturates instead of overflowing
        (1e30, 0x7BFF),
        (2.0 ** -14, 0x0400),              # smallest normal
        (2.0 ** -24, 0x0001),              # smallest subnormal
        (2.0 ** -25, 0x0000),              # tie between 0 and 2^-24: even (zero)
        (3 * 2.0 ** -26, 0x0001),          # 0.75 * 2^-24 rounds up
        (0.0, 0x0000),
    ]
    for x, bits in cases:
        got = int(i4.f32_to_f16_satfinite(np.array([x], np.float32))[0])
        assert got == bits, (x, hex(got), hex(bits))
        assert brute.f16_round(float(np.float32(x))) == float(i4.f16_to_f32(np.array([bits], np.uint16))[0])


def test_packing_is_twos_complement_low_nibble_first():
    codes = np.array([-8, -1, 0, 7, 3, -3], np.int8)
    packed = i4.pack_int4(codes)
    assert packed.tolist() == [0xF8, 0x70, 0xD3]
    assert np.array_equal(i4.unpack_int4(packed), codes)


def test_tie_cases_round_half_to_even():
    # amax = 7 gives s = 7 / 7 = 1 exactly, so v / s = v
    v = np.zeros(64, np.float32)
    vals = [7.0, 0.5, 1.5, 2.5, 3.5, -0.5, -1.5, -2.5, 6.5, -6.5, -7.0, 4.5, 0.49999997]
    want = [7, 0, 2, 2, 4, 0, -2, -2, 6, -6, -7, 4, 0]
    v[:len(vals)] = vals
    codes, s = i4.quantize_groups(v[None, :])
    assert int(s[0, 0]) == 0x3C00
    assert codes[0, :len(vals)].tolist() == want
    assert np.all(codes[0, len(vals):] == 0)


def test_representable_group_roundtrip():
    rng = np.random.default_rng(7)
    for _ in range(50):
        q = rng.integers(-7, 8, size=64)
        q[rng.integers(0, 64)] = 7 * rng.choice([-1, 1])          # max |q| = 7
        s_bits = np.uint16(rng.integers(0x0400, 0x7800))           # normal fp16 scale
        s = i4.f16_to_f32(np.array([s_bits]))[0]
        v = (q.astype(np.float32) * s).astype(np.float32)         # exact: <= 14 bits
        codes, sb = i4.quantize_groups(v[None, :])
        assert int(sb[0, 0]) == int(s_bits)
        assert np.array_equal(codes[0], q.astype(np.int8))


def test_power_of_two_homogeneity():
    rng = np.random.default_rng(8)
    v = rng.standard_normal((20, 128)).astype(np.float32)
    c0, s0 = i4.quantize_groups(v)
    for k in (-4, -1, 3, 7):
        c1, s1 = i4.quantize_groups((v * np.float32(2.0 ** k)).astype(np.float32))
        assert np.array_equal(c1, c0)
        assert np.array_equal(i4.f16_to_f32(s1), i4.f16_to_f32(s0) * np.float32(2.0 ** k))


def test_error_bound_and_range():
    rng = np.random.default_rng(9)
    v = rng.standard_normal((64, 256)).astype(np.float32)
    v[:, rng.choice(256, 5, replace=False)] *= 40
    codes, s = i4.quantize_groups(v)
    assert codes.min() >= -7 and codes.max() <= 7          # -8 needs a saturated scale
    deq = i4.dequantize_int4(i4.pack_int4(codes), s)
    sf = np.repeat(i4.f16_to_f32(s).astype(np.float64), 64, axis=1)
    assert np.all(np.abs(deq - v) <= sf * (0.5 + 2.0 ** -20))
    # the scale is within half an fp16 ulp (relative 2^-11) of amax / 7
    amax = np.abs(v.reshape(64, 4, 64)).max(axis=-1).astype(np.float64)
    assert np.all(np.abs(i4.f16_to_f32(s) - amax / 7) <= amax / 7 * 2.0 ** -11 * (1 + 1e-6))


def test_zero_and_saturated_groups():
    v = np.zeros((3, 64), np.float32)
    v[1, 0], v[1, 1], v[1, 2] = 1e6, -1e6, 1.0
    v[2, 5] = 1e-30                                        # amax / 7 below half of 2^-24
    codes, s = i4.quantize_groups(v)
    assert int(s[0, 0]) == 0 and np.all(codes[0] == 0)
    assert int(s[1, 0]) == 0x7BFF
    assert codes[1, :3].tolist() == [7, -8, 0]            # 1e6 / 65504 = 15.3 -> clamped
    assert int(s[2, 0]) == 0 and np.all(codes[2] == 0)     # s == 0: codes are 0


@pytest.mark.parametrize("M,N,K,r", [(1, 1, 64, 0), (3, 16, 64, 1), (16, 3, 128, 3),
                                     (5, 8, 128, 4), (2, 5, 64, 0)])
def test_brute_force_twin_int4(M, N, K, r):
    rng = np.random.default_rng(2000 + M * 100 + N * 10 + K + r)
    X = gen.random_bf16(rng, (M, K))
    X[:, 0] = gen.to_bf16_bits(gen.bf16_bits_to_f32(X[:, 0]).astype(np.float64) * 30)
    W = gen.random_bf16(rng, (N, K), 0.05)
    bias = gen.random_bf16(rng, (N,), 0.01)
    lam = gen.calibrate_lambda(X, W)
    w_hat = ref.smooth_weight(W, lam)
    if r:
        L1, L2, _ = ref.svd_split(w_hat, r)
    else:
        L1 = np.zeros((K, 0), np.uint16)
        L2 = np.zeros((0, N), np.uint16)
    _, wc, ws = i4.residual_quantize_int4(w_hat, L1, L2)
    prep = dict(inv_lambda=ref.inv_lambda_of(lam), L1=L1, L2t=np.ascontiguousarray(L2.T),
                w_codes=wc, w_scales=ws, bias=bias)
    o = i4.linear_forward_int4(X, prep)
    b = brute.forward_int4(X.tolist(), W.tolist(), lam.tolist(), bias.tolist(),
                           L1.tolist(), L2.tolist())
    assert np.array_equal(i4.unpack_int4(o["x_codes"]), np.array(b["x_codes"], np.int8))
    assert np.array_equal(i4.f16_to_f32(o["x_scales"]), np.array(b["x_scales"], np.float32))
    assert np.array_equal(i4.unpack_int4(wc), np.array(b["w_codes"], np.int8))
    assert np.array_equal(i4.f16_to_f32(ws), np.array(b["w_scales"], np.float32))
    if r:
        assert np.array_equal(ref.bf16_to_f64(o["D"]), np.array(b["D"]))
    y_b = np.array(b["Y64"])
    assert np.max(np.abs(o["Y64"] - y_b)) <= 1e-12 * max(np.abs(y_b).max(), 1e-30)


def test_forward_r0_lambda1_is_plain_int4_gemm():
    """r = 0, lambda = 1: Y = deq(Q(X)) deq(Q(W))^T + b, composed by explicit loops."""
    rng = np.random.default_rng(32)
    M, N, K = 4, 6, 128
    X = gen.random_bf16(rng, (M, K))
    W = gen.random_bf16(rng, (N, K), 0.1)
    bias = gen.random_bf16(rng, (N,), 0.01)
    lam = np.ones(K, np.float32)
    z1, z2 = np.zeros((K, 0), np.uint16), np.zeros((0, N), np.uint16)
    _, wc, ws = i4.residual_quantize_int4(ref.smooth_weight(W, lam), z1, z2)
    prep = dict(inv_lambda=ref.inv_lambda_of(lam), L1=z1, L2t=z2.T, w_codes=wc, w_scales=ws,
                bias=bias)
    y = i4.linear_forward_int4(X, prep)["Y64"]
    cx, sx = i4.quantize_groups(gen.bf16_bits_to_f32(X))
    cw, sw = i4.quantize_groups(gen.bf16_bits_to_f32(W))
    sxf, swf = i4.f16_to_f32(sx), i4.f16_to_f32(sw)
    want = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for g in range(K // 64):
                isum = 0
                for k in range(64 * g, 64 * g + 64):
                    isum += int(cx[m, k]) * int(cw[n, k])          # exact integer group sum
                acc += float(sxf[m, g]) * float(swf[n, g]) * isum
            want[m, n] = acc + float(ref.bf16_to_f64(bias[n:n + 1])[0])
    assert np.max(np.abs(y - want)) <= 1e-12 * np.abs(want).max()


def test_quality_sanity_int4_error_falls_with_rank_and_smoothing():
    """Not a parity pin: the INT4 layer must do the method's job as well."""
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
        prep = i4.prepare_weight_int4(W, lam_, None, r)
        yq = i4.linear_forward_int4(X, prep)["Y64"]
        return np.linalg.norm(yq - y) / np.linalg.norm(y)

    e0, e8, e32 = err(lam, 0), err(lam, 8), err(lam, 32)
    assert e32 < e8 < e0
    assert e32 < err(np.ones(K, np.float32), 32)
