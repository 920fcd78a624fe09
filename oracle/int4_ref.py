"""CPU oracle of the INT4 variant of the SVDQuant W4A4 layer (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may use it; nothing in the product imports it.

What the pages fix: the same layer exists in two 4-bit formats, NVFP4 for
Blackwell and INT4 for the earlier NVIDIA generations (Turing, Ampere, Ada)
(chaosnode.de "Nunchaku Lite: 4-Bit Diffusion-Inferenz direkt in Diffusers",
section "Hardware-Support"; imaginepro.ai "Nunchaku 4-Bit Diffusion
Inference in Diffusers: A Practical Guide", table "Supported quantisation
methods": svdq_w4a4 in INT4).  The pages say nothing else about the INT4
format, so every detail below is a reading (listed with the others):

  R15 INT4 codes are signed two's-complement 4-bit integers in [-8, 7], one
      scale per group of 64 consecutive elements along K, packed like NVFP4
      (element 2j in the low nibble of byte j).
  R16 Group quantiser on 64 values v: a = max|v|; s = fp16_RNE(min(f32(a / 7),
      65504)) (an f32 division, then a saturating rounding to half precision);
      q_i = clamp(RNE(f32(v_i / s)), -8, 7) with an IEEE f32 division, and
      q_i = 0 where s == 0.  Because |v_i / s| <= 7 (1 + 2^-11) the clamp
      only acts when s saturated; -8 is never produced otherwise.
  R17 Scales are fp16 bit patterns, stored logically as [rows][K/64].
  R18 Y = bf16_RNE(sum_k deq(qx)_mk deq(qR)_nk + sum_j D_mj bf16(L2)_jn + bias_n)
      in f64, deq(q) = q s.  Smoothing, the rank-r split, the residual and D
      are those of the NVFP4 layer (readings R1-R5, R8): only the 4-bit format
      of Q4 changes.
"""
from __future__ import annotations

import numpy as np

from . import svdq_ref as ref

__all__ = ["GROUP", "FP16_MAX", "f32_to_f16_satfinite", "f16_to_f32", "quantize_groups",
           "dequantize_int4", "residual_quantize_int4", "prepare_weight_int4",
           "quantize_act_int4", "linear_forward_int4", "pack_int4", "unpack_int4"]

GROUP = 64
FP16_MAX = np.float32(65504.0)


def f32_to_f16_satfinite(x: np.ndarray) -> np.ndarray:
    """fp16 bit patterns (uint16) of non-negative float32 values: IEEE RNE
    (NumPy's float16 conversion), clamped first to the largest finite fp16."""
    x = np.minimum(np.asarray(x, dtype=np.float32), FP16_MAX)
    return x.astype(np.float16).view(np.uint16)


def f16_to_f32(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> exact float32 values."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float32)


def quantize_groups(v: np.ndarray):
    """Quantise rows of float32 values in groups of 64 along the last axis (R16).

    Returns (codes, scales): codes int8 [..., K] in [-8, 7] (unpacked), scales
    uint16 [..., K/64] (fp16 bit patterns).
    """
    v = np.asarray(v, dtype=np.float32)
    K = v.shape[-1]
    if K % GROUP:
        raise ValueError("K must be a multiple of 64")
    grp = v.reshape(v.shape[:-1] + (K // GROUP, GROUP))
    amax = np.abs(grp).max(axis=-1)                                  # exact
    s_bits = f32_to_f16_satfinite(np.float32(amax) / np.float32(7.0))  # f32 division first
    s = f16_to_f32(s_bits)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (grp / s[..., None]).astype(np.float32)                  # IEEE f32 division
    q = np.clip(np.rint(q), -8, 7)                                   # rint: ties to even
    q = np.where((s == 0)[..., None], 0, q)
    return q.astype(np.int8).reshape(v.shape), s_bits


def pack_int4(codes: np.ndarray) -> np.ndarray:
    """[..., K] int codes in [-8, 7] -> [..., K/2] bytes of two's-complement nibbles."""
    return ref.pack_nibbles(np.asarray(codes).astype(np.int16) & 0xF)


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] int8 codes (nibbles sign-extended)."""
    n = ref.unpack_nibbles(packed).astype(np.int16)
    return np.where(n >= 8, n - 16, n).astype(np.int8)


def dequantize_int4(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float64 values q s of packed INT4 rows with logical [rows][K/64] fp16 scales."""
    q = unpack_int4(packed).astype(np.float64)
    s = f16_to_f32(scales).astype(np.float64)
    K = q.shape[-1]
    return (q.reshape(q.shape[:-1] + (K // GROUP, GROUP)) * s[..., None]).reshape(q.shape)


def residual_quantize_int4(w_hat: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray):
    """R = f32(What - (bf16 L1 . bf16 L2)^T) (reading R5), then INT4 along K.

    Returns (R f32 N x K, packed codes N x K/2, fp16 scales N x K/64).
    """
    R = ref.residual(w_hat, ref.bf16_to_f64(L1_bits), ref.bf16_to_f64(L2_bits)).astype(np.float32)
    codes, scales = quantize_groups(R)
    return R, pack_int4(codes), scales


def prepare_weight_int4(w_bits: np.ndarray, lam: np.ndarray, bias_bits, r: int) -> dict:
    """Offline preparation in the INT4 format: smoothing, rank-r split, residual pack."""
    inv = ref.inv_lambda_of(lam)
    w_hat = ref.smooth_weight(w_bits, lam)
    L1, L2, sig = ref.svd_split(w_hat, r)
    R, codes, scales = residual_quantize_int4(w_hat, L1, L2)
    return dict(inv_lambda=inv, w_hat=w_hat, L1=L1, L2=L2, L2t=np.ascontiguousarray(L2.T),
                sigma=sig, R=R, w_codes=codes, w_scales=scales,
                bias=None if bias_bits is None else np.asarray(bias_bits, dtype=np.uint16), r=r)


def quantize_act_int4(x_bits: np.ndarray, inv_lambda: np.ndarray, L1_bits) -> dict:
    """Activation side in the INT4 format: Xhat, its codes/scales and D (R8)."""
    x_hat = ref.smooth_act(x_bits, inv_lambda)
    codes, scales = quantize_groups(x_hat)
    out = dict(x_hat=x_hat, x_codes=pack_int4(codes), x_scales=scales)
    if L1_bits is not None and np.asarray(L1_bits).shape[-1] > 0:
        out["D"], out["D_abs"] = ref.lowrank_down(x_hat, L1_bits)
    else:
        out["D"] = np.zeros((x_hat.shape[0], 0), dtype=np.uint16)
        out["D_abs"] = np.zeros((x_hat.shape[0], 0))
    return out


def linear_forward_int4(x_bits: np.ndarray, prep: dict, rows=None) -> dict:
    """Y of the INT4 layer (R18) for a weight from prepare_weight_int4 (or an
    exported one with the same fields).  ``rows`` restricts the token rows."""
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    if rows is not None:
        x_bits = x_bits[np.asarray(rows)]
    act = quantize_act_int4(x_bits, prep["inv_lambda"], prep["L1"])
    y = dequantize_int4(act["x_codes"], act["x_scales"]) @ \
        dequantize_int4(prep["w_codes"], prep["w_scales"]).T
    if np.asarray(prep["L1"]).shape[-1] > 0:
        y = y + ref.bf16_to_f64(act["D"]) @ ref.bf16_to_f64(prep["L2t"]).T
    if prep.get("bias") is not None:
        y = y + ref.bf16_to_f64(prep["bias"])[None, :]
    return dict(Y=ref.f64_to_bf16(y), Y64=y, **act)
