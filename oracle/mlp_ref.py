"""CPU oracle of the fused MLP pair (TEST INFRASTRUCTURE ONLY).

The engine the pages describe fuses model-specific kernels, among them a
GELU/MLP path (chaosnode.de "Nunchaku Lite: 4-Bit Diffusion-Inferenz direkt
in Diffusers", section "Nunchaku Lite vs. Original").  For a DiT MLP the pair
is: up-projection linear, GELU, down-projection linear, both linears being
SVDQuant W4A4 layers.  The fused kernels have to reproduce this composition;
this module states it.  Only ``tests/`` may import it.

Readings (the pages give no formula for the pair):
  R19 The hidden activation is H = bf16_RNE(gelu_tanh(Y_up)), with Y_up the
      up-projection's bf16 output and gelu_tanh(y) = y/2 (1 + tanh(sqrt(2/pi)
      (y + 0.044715 y^3))), its value computed in float64 and rounded once.
      The value is computed through the identity 1 + tanh u = 2 / (1 +
      e^{-2u}), i.e. gelu_tanh(y) = y / (1 + e^{-2u}): the same function,
      without the cancellation of 1 + tanh u, which in float64 loses every
      significant digit once tanh u is within 1e-16 of -1 (y below about
      -5.5, where H is still a normal bf16 number down to about y = -10).  The
      down-projection then runs on H exactly as a standalone layer would
      (smoothing by its own lambda, NVFP4 or INT4 quantisation, its own D).
      A fused kernel that evaluates GELU in float32 may differ from H by one
      bf16 step where the float64 value lies next to a rounding boundary; its
      downstream codes are then compared given its own H.
"""
from __future__ import annotations

import math

import numpy as np

from . import int4_ref
from . import svdq_ref as ref

__all__ = ["gelu_tanh_f64", "mlp_hidden", "mlp_pair_forward"]

_C = math.sqrt(2.0 / math.pi)


def gelu_tanh_f64(y: np.ndarray) -> np.ndarray:
    """tanh-approximated GELU in float64, as y / (1 + exp(-2u)) (R19)."""
    y = np.asarray(y, dtype=np.float64)
    u = _C * (y + 0.044715 * y ** 3)
    with np.errstate(over="ignore"):
        return y / (1.0 + np.exp(-2.0 * u))


def mlp_hidden(y_up_bits: np.ndarray) -> np.ndarray:
    """H = bf16(gelu_tanh(Y_up)) for the up-projection's bf16 output (R19)."""
    return ref.f64_to_bf16(gelu_tanh_f64(ref.bf16_to_f64(y_up_bits)))


def mlp_pair_forward(x_bits: np.ndarray, prep_up: dict, prep_down: dict, fmt: str = "nvfp4") -> dict:
    """Up-projection, GELU, down-projection (R19), each linear in ``fmt``.

    ``prep_up`` / ``prep_down`` are prepared weights of the two linears (the
    dicts of prepare_weight / prepare_weight_int4, or exported ones).  Returns
    the up-projection's output, H, and the down-projection's result dict."""
    forward = int4_ref.linear_forward_int4 if fmt == "int4" else ref.linear_forward
    up = forward(x_bits, prep_up)
    H = mlp_hidden(up["Y"])
    down = forward(H, prep_down)
    return dict(Y_up=up["Y"], H=H, Y=down["Y"], Y64=down["Y64"], down=down)
