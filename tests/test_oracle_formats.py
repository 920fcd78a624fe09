"""Pins of the oracle's number formats against closed forms and hand-derived values.

Every check here compares the oracle (table search, bit tricks) with something
independent of it: the hand-derived fixtures in tests/golden, closed-form
roundings written from the format definitions (brute-force twin), or exact
round trips of representable values.
"""
import math
import os

import numpy as np
import pytest

from oracle import brute
from oracle import svdq_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rounding():
    rows = []
    with open(os.path.join(GOLDEN, "e2m1_e4m3_rounding.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            kind, val, code = line.split()[:3]
            rows.append((kind, float(val), int(code, 16)))
    return rows


@pytest.mark.parametrize("kind,val,code", _golden_rounding())
def test_golden_rounding(kind, val, code):
    x = np.array([val], dtype=np.float32)
    if kind == "e2m1":
        assert int(ref.e2m1_encode(x)[0]) == code
        assert brute.e2m1_code(brute.e2m1_round(float(x[0]))) == code
    else:
        assert int(ref.e4m3_encode(x)[0]) == code
        assert brute.e4m3_code(brute.e4m3_round(float(x[0]))) == code


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = ref.e2m1_decode(codes).astype(np.float32)
    # -0.0 must keep its sign so code 8 comes back
    vals[8] = np.float32(-0.0)
    assert np.array_equal(ref.e2m1_encode(vals), codes)


def test_e4m3_roundtrip_all_codes():
    codes = np.arange(127, dtype=np.uint8)
    vals = ref.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(ref.e4m3_encode(vals), codes)
    assert ref.e4m3_decode(np.array([0x7E], np.uint8))[0] == 448.0
    assert ref.e4m3_decode(np.array([0x01], np.uint8))[0] == 2.0 ** -9
    assert ref.e4m3_decode(np.array([0x08], np.uint8))[0] == 2.0 ** -6
    # strictly increasing: codes order the values
    assert np.all(np.diff(ref.e4m3_table()) > 0)


def _sweep_points(grid_vals, rng, n_random=20000, hi=None):
    """Grid points, midpoints, their f32 neighbours, plus log-uniform randoms."""
    g = np.asarray(sorted(set(grid_vals)), dtype=np.float64)
    mids = (g[:-1] + g[1:]) / 2
    pts = np.concatenate([g, mids]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    hi = hi if hi is not None else g[-1] * 4
    rnd = np.exp(rng.uniform(np.log(g[1] / 8), np.log(hi), n_random)).astype(np.float32)
    return np.concatenate([pts, up, dn, rnd, np.array([hi * 1e3], np.float32)])


def test_e2m1_closed_form_sweep():
    rng = np.random.default_rng(11)
    x = _sweep_points(ref.E2M1_VALUES, rng)
    x = np.concatenate([x, -x])
    got = ref.e2m1_encode(x)
    want = np.array([brute.e2m1_code(brute.e2m1_round(float(v))) for v in x], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e4m3_closed_form_sweep():
    rng = np.random.default_rng(12)
    x = _sweep_points(ref.e4m3_table(), rng, hi=2000.0)
    got = ref.e4m3_encode(x)
    want = np.array([brute.e4m3_code(brute.e4m3_round(float(v))) for v in x], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_bf16_rounding_against_f32_bit_rule_and_closed_form():
    rng = np.random.default_rng(13)
    # values that are exactly float32: f64->bf16 must equal the f32 bit rule
    f = (rng.standard_normal(50000) * np.exp(rng.uniform(-30, 30, 50000))).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rule = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(ref.f64_to_bf16(f.astype(np.float64)), rule)
    # arbitrary float64 values (not float32-exact): closed form via frexp
    d = rng.standard_normal(5000) * np.exp(rng.uniform(-20, 20, 5000))
    got = ref.bf16_to_f64(ref.f64_to_bf16(d))
    want = np.array([brute.bf16_round(float(v)) for v in d])
    assert np.array_equal(got, want)
    # explicit ties: 1 + 2^-8 -> 1 (even), 1 + 3*2^-8 -> 1 + 2^-6 (even)
    t = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])
    assert list(ref.bf16_to_f64(ref.f64_to_bf16(t))) == [1.0, 1 + 2.0 ** -6, -1.0]
    # the rounding is a single rounding from f64: 1 + 2^-8 + 2^-40 rounds up
    assert ref.bf16_to_f64(ref.f64_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40])))[0] == 1 + 2.0 ** -7
    # bf16 subnormal range
    s = np.array([3 * 2.0 ** -134, 5 * 2.0 ** -134, 2.0 ** -130])
    assert list(ref.bf16_to_f64(ref.f64_to_bf16(s))) == [2 * 2.0 ** -133, 2 * 2.0 ** -133, 2.0 ** -130]


def test_bf16_to_f64_is_exact_decoding():
    bits = np.array([0x3F80, 0xBF80, 0x4040, 0x0000, 0x8000, 0x7F7F], np.uint16)
    want = [1.0, -1.0, 3.0, 0.0, -0.0, 3.3895313892515355e38]
    got = ref.bf16_to_f64(bits)
    assert list(got) == want
    assert math.copysign(1, got[4]) < 0
