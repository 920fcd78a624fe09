"""Mutation checks of the pins: each test plants one plausible mistake in the
oracle (on the CPU, through monkeypatch) and requires that at least one of the
named pins fails.  A pin set that lets a planted mistake through is too weak."""
import numpy as np
import pytest

from oracle import int4_ref as i4
from oracle import svdq_ref as ref

import test_oracle_int4 as pins4
import test_oracle_quant as pins


def _some_pin_fails(tests):
    failed = []
    for t in tests:
        try:
            t()
        except AssertionError:
            failed.append(t.__name__)
    return failed


NVFP4_PINS = [pins.test_packing_order, pins.test_representable_block_roundtrip,
              pins.test_power_of_two_scaling_invariance, pins.test_zero_block_and_tiny_block,
              pins.test_forward_r0_lambda1_is_plain_nvfp4_gemm]
INT4_PINS = [pins4.test_packing_is_twos_complement_low_nibble_first, pins4.test_tie_cases_round_half_to_even,
             pins4.test_representable_group_roundtrip, pins4.test_power_of_two_homogeneity,
             pins4.test_error_bound_and_range, pins4.test_zero_and_saturated_groups,
             pins4.test_forward_r0_lambda1_is_plain_int4_gemm]


def _swapped_nibbles(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return ((c[..., 0::2] << 4) | c[..., 1::2]).astype(np.uint8)


def _unpack_swapped(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p >> 4
    out[..., 1::2] = p & 0xF
    return out


def test_nvfp4_nibble_order_swapped(monkeypatch):
    monkeypatch.setattr(ref, "pack_nibbles", _swapped_nibbles)
    monkeypatch.setattr(ref, "unpack_nibbles", _unpack_swapped)
    assert _some_pin_fails(NVFP4_PINS)


def test_nvfp4_scale_from_amax_over_4(monkeypatch):
    real = ref.e4m3_encode
    monkeypatch.setattr(ref, "e4m3_encode", lambda x: real(np.asarray(x, np.float32) * np.float32(1.5)))
    assert _some_pin_fails(NVFP4_PINS)


def test_nvfp4_sign_bit_dropped(monkeypatch):
    real = ref.e2m1_encode
    monkeypatch.setattr(ref, "e2m1_encode", lambda x: real(np.abs(np.asarray(x, np.float32))))
    assert _some_pin_fails(NVFP4_PINS)


def test_nvfp4_grid_with_a_wrong_top_value(monkeypatch):
    monkeypatch.setattr(ref, "E2M1_VALUES", np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0]))
    assert _some_pin_fails(NVFP4_PINS)


def test_int4_scale_from_amax_over_8(monkeypatch):
    real = i4.f32_to_f16_satfinite
    monkeypatch.setattr(i4, "f32_to_f16_satfinite",
                        lambda x: real(np.asarray(x, np.float32) * np.float32(7.0 / 8.0)))
    assert _some_pin_fails(INT4_PINS)


def test_int4_rounding_half_up(monkeypatch):
    monkeypatch.setattr(i4.np, "rint", lambda x: np.floor(np.asarray(x) + 0.5))
    try:
        assert _some_pin_fails(INT4_PINS)
    finally:
        monkeypatch.undo()


def test_int4_sign_extension_off_by_eight(monkeypatch):
    def unpack(packed):
        n = ref.unpack_nibbles(packed).astype(np.int16)
        return np.where(n >= 8, n - 8, n).astype(np.int8)
    monkeypatch.setattr(i4, "unpack_int4", unpack)
    assert _some_pin_fails(INT4_PINS)


def test_unmutated_oracle_passes_every_pin():
    assert _some_pin_fails(NVFP4_PINS + INT4_PINS) == []
