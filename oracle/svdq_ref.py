"""CPU oracle for the SVDQuant W4A4 linear layer (TEST INFRASTRUCTURE ONLY).

This is a plain, slow, obviously-correct NumPy restatement of what the layer
computes.  It shares no code with the CUDA path and nothing in the product
imports it: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm may use it.

What the pages fix (all in prose; no page prints a formula or a number for a
single layer):
  * W4A4: weights and activations are both 4-bit; activation outliers are
    moved ("migrated") into the weights, the hard part becomes a 16-bit
    low-rank branch, the rest is quantised to 4 bits
    (aiphreaks.com "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
    section "Technical Breakdown and Performance Metrics";
    chaosnode.de "Nunchaku Lite: 4-Bit Diffusion-Inferenz direkt in Diffusers",
    section "Die Technik: SVDQuant").
  * The weight is split into a low-rank component plus a residual; most work
    runs on 4-bit tensor cores, the low-rank correction in higher precision
    (imaginepro.ai "Nunchaku 4-Bit Diffusion Inference in Diffusers: A
    Practical Guide", section "Under the Hood: 4-Bit Quantization for
    Diffusion Models").
  * NVFP4 is the 4-bit format on Blackwell, B200 included (chaosnode.de,
    section "Hardware-Support"); rank 32 (watch-ia.com, checkpoint name
    "...nvfp4_r32...").

The layer follows this formula (the pages describe it in words only):
    Y = Xhat L1 L2 + Q4(Xhat) Q4(R)^T + b,   Xhat = X diag(1/lambda),
    R = diag(lambda) W - (L1 L2)^T           (read with W as K x N, see below),
NVFP4 = E2M1 codes with one E4M3 scale per 16 consecutive elements along K.

Readings where the pages are silent (numbered R1-R9, the same numbers the kernels cite):
  R1  W is stored N x K (nn.Linear layout, Y = X W^T).  The residual formula
      is read with W taken K x N there, so What = W diag(lambda) (N x K),
      the SVD is of What^T (K x N), L1 L2 ~= What^T and R = What - (L1 L2)^T
      is N x K: its NVFP4 blocks then run along K as the format requires.
  R2  inv_lambda = f32(1/lambda) is stored, and smoothing multiplies by it:
      Xhat = f32(X * inv_lambda) (one rounded f32 multiply).
  R3  What = f32(W * lambda) (one rounded f32 multiply).
  R4  SVD split: L1 = U_r diag(sigma_r) (K x r), L2 = V_r^T (r x N); each
      singular pair is sign-normalised so that the largest-|.| entry of u_i
      is positive; L1 and L2 are stored as bf16 (RNE).
  R5  R_nk = f32(What_nk - sum_j bf16(L1)_kj bf16(L2)_jn), the sum taken in
      f64 in increasing j: the residual absorbs the bf16 rounding of L1, L2.
  R6  Block quantiser on 16 values v: a = max|v|; s = E4M3_RNE_satfinite(
      f32(a / 6)); q_i = E2M1_RNE_satfinite(f32(v_i / s)), with v_i / s
      replaced by copysign(0, v_i) when s == 0.  The sign bit of E2M1 is
      kept, so a negative value that rounds to zero is code 0x8.
  R7  Packing: element 2j of a row goes to the low nibble of byte j, element
      2j+1 to the high nibble.  Scales are stored logically as [rows][K/16].
  R8  D = bf16_RNE(sum_k bf16(Xhat)_mk bf16(L1)_kj) summed in f64: the
      low-rank branch takes bf16 operands (the pages' "16-bit" branch).
  R9  Y = bf16_RNE(sum_k deq(qx)_mk deq(qR)_nk + sum_j D_mj bf16(L2)_jn
      + bias_n), all in f64, one final rounding.

Values are passed as NumPy arrays: bf16 as uint16 bit patterns, float32 as
np.float32, codes/scales as uint8.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_to_f64", "f64_to_bf16", "E2M1_VALUES", "e4m3_table", "e4m3_encode",
    "e4m3_decode", "e2m1_encode", "e2m1_decode", "quantize_blocks",
    "pack_nibbles", "unpack_nibbles", "dequantize", "inv_lambda_of",
    "smooth_act", "smooth_weight", "svd_split", "residual_quantize",
    "prepare_weight", "quantize_act", "lowrank_down", "linear_forward",
]

# ---------------------------------------------------------------------------
# bf16 <-> f64
# ---------------------------------------------------------------------------


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 with round-to-nearest-even (one rounding).

    Normal range: keep 8 significant bits of the float64 significand with RNE
    on the 45 discarded bits.  Below 2^-126 (bf16 subnormals) round to a
    multiple of 2^-133 with ties to even.  NaN/Inf are not expected.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    tiny = np.abs(x) < 2.0 ** -126
    # normal path on the float64 bit pattern
    u = x.view(np.uint64).copy()
    lsb = (u >> np.uint64(45)) & np.uint64(1)
    u = (u + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    v = u.view(np.float64).astype(np.float32)       # exact: <= 8 significant bits
    out_n = (v.view(np.uint32) >> 16).astype(np.uint16)
    # subnormal path: integer multiple of 2^-133, RNE via rint
    m = np.rint(x * 2.0 ** 133)                     # exact scaling, rint is ties-to-even
    v_s = (m * 2.0 ** -133).astype(np.float32)      # representable exactly
    out_s = (v_s.view(np.uint32) >> 16).astype(np.uint16)
    out[...] = np.where(tiny, out_s, out_n)
    return out


# ---------------------------------------------------------------------------
# E4M3 (scale) and E2M1 (element) conversions, table driven
# ---------------------------------------------------------------------------

E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])  # codes 0..7


def e4m3_table() -> np.ndarray:
    """Values of the 127 finite non-negative E4M3 codes 0x00..0x7E.

    E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0
    is subnormal (m/8 * 2^-6); 0x7F is NaN, so the largest finite is
    0x7E = 1.75 * 2^8 = 448.
    """
    vals = np.empty(127)
    for c in range(127):
        e, m = c >> 3, c & 7
        vals[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_table()


def _nearest_even(x: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to x (x >= 0, grid ascending, index = code).

    Exact in float64 (all inputs are float32 values, all grid points and their
    midpoints are float64-exact).  Ties go to the even code.  Values above the
    last grid point saturate to it (satfinite).
    """
    x = np.asarray(x, dtype=np.float64)
    hi = np.searchsorted(grid, x, side="left")          # grid[hi-1] < x <= grid[hi]
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    dlo = x - grid[lo]
    dhi = grid[hi] - x
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(x >= grid[-1], len(grid) - 1, idx)
    idx = np.where(x <= grid[0], 0, idx)
    return idx


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """E4M3 code (uint8) of non-negative float32 values, RNE, satfinite (448)."""
    x = np.asarray(x, dtype=np.float32)
    if np.any(x < 0) or np.any(~np.isfinite(x)):
        raise ValueError("e4m3_encode: scales must be finite and non-negative")
    return _nearest_even(x, _E4M3).astype(np.uint8)


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    if np.any((code & 0x7F) == 0x7F):
        raise ValueError("e4m3_decode: NaN code")
    mag = _E4M3[code & 0x7F]
    return np.where(code & 0x80, -mag, mag)


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """E2M1 code (4 bits in a uint8) of float32 values: sign bit 0x8 kept, RNE,
    magnitudes above 6 saturate to 6."""
    x = np.asarray(x, dtype=np.float32)
    if np.any(~np.isfinite(x)):
        raise ValueError("e2m1_encode: non-finite input")
    mag = _nearest_even(np.abs(x).astype(np.float64), E2M1_VALUES).astype(np.uint8)
    sign = np.signbit(x).astype(np.uint8) << 3
    return (sign | mag).astype(np.uint8)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


# ---------------------------------------------------------------------------
# NVFP4 block quantiser (reading R6) and packing (R7)
# ---------------------------------------------------------------------------


def quantize_blocks(v: np.ndarray):
    """Quantise rows of float32 values in blocks of 16 along the last axis.

    Returns (codes, scales): codes uint8 [..., K] (one 4-bit code per element,
    unpacked), scales uint8 [..., K/16] (E4M3 codes).
    """
    v = np.asarray(v, dtype=np.float32)
    K = v.shape[-1]
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    blk = v.reshape(v.shape[:-1] + (K // 16, 16))
    amax = np.abs(blk).max(axis=-1)                              # exact (f32)
    s_code = e4m3_encode(np.float32(amax) / np.float32(6.0))     # f32 division, then RNE
    s = e4m3_decode(s_code).astype(np.float32)                   # exact
    with np.errstate(divide="ignore", invalid="ignore"):
        q = blk / s[..., None]                                    # f32 division (IEEE)
    zero = (s == 0)[..., None]
    q = np.where(zero, np.copysign(np.float32(0), blk), q).astype(np.float32)
    codes = e2m1_encode(q).reshape(v.shape)
    return codes, s_code


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., K] 4-bit codes -> [..., K/2] bytes, element 2j in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """float64 values of packed NVFP4 rows with logical [rows][K/16] scales."""
    codes = unpack_nibbles(packed)
    vals = e2m1_decode(codes)
    s = e4m3_decode(scales)
    K = vals.shape[-1]
    return (vals.reshape(vals.shape[:-1] + (K // 16, 16)) * s[..., None]).reshape(vals.shape)


# ---------------------------------------------------------------------------
# Smoothing (R2, R3)
# ---------------------------------------------------------------------------


def column_absmax(a_bits: np.ndarray) -> np.ndarray:
    """max over rows of |A[:, k]| for a bf16 matrix (float32; exact)."""
    return np.abs(bf16_to_f64(a_bits)).max(axis=0).astype(np.float32)


def calibrate_lambda(x_absmax: np.ndarray, w_bits: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """Smoothing factors from calibration statistics (offline step).

    The pages move each input channel's activation outliers into the weight
    (chaosnode.de "Nunchaku Lite ...", section "Die Technik: SVDQuant") and
    calibrate offline (watch-ia.com, last paragraphs), but give no formula.
    Reading: lambda_k = x_k^alpha / w_k^(1-alpha) with x_k = max|X[:, k]| over
    the calibration activations, w_k = max|W[:, k]|, in float64, rounded once to
    float32; alpha = 0.5 (the inputs' recipe) is evaluated as sqrt(x_k / w_k);
    lambda_k = 1 where either maximum is 0.
    """
    x = np.asarray(x_absmax, dtype=np.float64)
    w = column_absmax(w_bits).astype(np.float64)
    lam = np.ones_like(x)
    ok = (x > 0) & (w > 0)
    if alpha == 0.5:
        lam[ok] = np.sqrt(x[ok] / w[ok])
    else:
        lam[ok] = np.power(x[ok], alpha) / np.power(w[ok], 1.0 - alpha)
    return lam.astype(np.float32)


def inv_lambda_of(lam: np.ndarray) -> np.ndarray:
    lam = np.asarray(lam, dtype=np.float32)
    return (np.float32(1.0) / lam).astype(np.float32)


def smooth_act(x_bits: np.ndarray, inv_lambda: np.ndarray, dtype=np.float32) -> np.ndarray:
    """Xhat = X diag(inv_lambda): column k of X is multiplied by inv_lambda[k].

    dtype=float32 is the layer's arithmetic (one rounded multiply); dtype=float64
    is used by the smoothing-identity pin.
    """
    x = bf16_to_f64(x_bits).astype(dtype)
    return (x * np.asarray(inv_lambda).astype(dtype)[None, :]).astype(dtype)


def smooth_weight(w_bits: np.ndarray, lam: np.ndarray, dtype=np.float32) -> np.ndarray:
    """What = W diag(lambda) for W stored N x K: column k scaled by lambda[k]."""
    w = bf16_to_f64(w_bits).astype(dtype)
    return (w * np.asarray(lam).astype(dtype)[None, :]).astype(dtype)


# ---------------------------------------------------------------------------
# Rank-r split (R4) and residual (R5)
# ---------------------------------------------------------------------------


def svd_split(w_hat: np.ndarray, r: int, round_bf16: bool = True):
    """Top-r SVD of What^T (K x N) in float64.

    Returns (L1, L2, sigma): L1 = U_r diag(sigma_r) (K x r), L2 = V_r^T (r x N),
    sigma = all singular values (descending).  With round_bf16, L1 and L2 are
    returned as bf16 bit patterns, else as float64.
    """
    a = np.asarray(w_hat, dtype=np.float64).T          # K x N
    K, N = a.shape
    if not 0 <= r <= min(K, N):
        raise ValueError("rank out of range")
    u, sig, vt = np.linalg.svd(a, full_matrices=False)
    u = u[:, :r].copy()
    vt = vt[:r, :].copy()
    for i in range(r):
        j = int(np.argmax(np.abs(u[:, i])))
        if u[j, i] < 0:
            u[:, i] = -u[:, i]
            vt[i, :] = -vt[i, :]
    L1 = u * sig[None, :r]
    L2 = vt
    if round_bf16:
        return f64_to_bf16(L1), f64_to_bf16(L2), sig
    return L1, L2, sig


def residual(w_hat: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """R = What - (L1 L2)^T, accumulated in float64 in increasing j (N x K).

    L1 (K x r) and L2 (r x N) are float64 values (already bf16-rounded when the
    layer's arithmetic is wanted).  The result stays float64.
    """
    K, r = L1.shape
    acc = np.zeros((L2.shape[1], K), dtype=np.float64)
    for j in range(r):
        acc += np.outer(L2[j, :], L1[:, j])      # bf16*bf16 products are exact
    return np.asarray(w_hat, dtype=np.float64) - acc


def residual_quantize(w_hat: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray):
    """R = f32(What - (bf16 L1 . bf16 L2)^T), then NVFP4 along K.

    Returns (R f32 N x K, packed codes N x K/2, scales N x K/16).
    """
    L1 = bf16_to_f64(L1_bits)
    L2 = bf16_to_f64(L2_bits)
    R = residual(w_hat, L1, L2).astype(np.float32)
    codes, scales = quantize_blocks(R)
    return R, pack_nibbles(codes), scales


def prepare_weight(w_bits: np.ndarray, lam: np.ndarray, bias_bits, r: int) -> dict:
    """Offline preparation of one linear: smoothing, rank-r split, residual pack."""
    inv = inv_lambda_of(lam)
    w_hat = smooth_weight(w_bits, lam)
    L1, L2, sig = svd_split(w_hat, r)
    R, codes, scales = residual_quantize(w_hat, L1, L2)
    return dict(inv_lambda=inv, w_hat=w_hat, L1=L1, L2=L2, L2t=np.ascontiguousarray(L2.T),
                sigma=sig, R=R, w_codes=codes, w_scales=scales,
                bias=None if bias_bits is None else np.asarray(bias_bits, dtype=np.uint16), r=r)


# ---------------------------------------------------------------------------
# Activation path and forward (R8, R9)
# ---------------------------------------------------------------------------


def lowrank_down(x_hat: np.ndarray, L1_bits: np.ndarray):
    """D = bf16(sum_k bf16(Xhat)_mk bf16(L1)_kj), f64 sum.  Returns (D bits, |.|-sum).

    The second value, sum_k |bf16(Xhat)_mk bf16(L1)_kj|, bounds the rounding
    error any fp32 accumulation of the same products can make.
    """
    xb = bf16_to_f64(f64_to_bf16(np.asarray(x_hat, dtype=np.float64)))
    L1 = bf16_to_f64(L1_bits)
    d = xb @ L1
    return f64_to_bf16(d), np.abs(xb) @ np.abs(L1)


def quantize_act(x_bits: np.ndarray, inv_lambda: np.ndarray, L1_bits) -> dict:
    """Activation side of the layer: Xhat, its NVFP4 codes/scales and D."""
    x_hat = smooth_act(x_bits, inv_lambda)
    codes, scales = quantize_blocks(x_hat)
    out = dict(x_hat=x_hat, x_codes=pack_nibbles(codes), x_scales=scales)
    if L1_bits is not None and np.asarray(L1_bits).shape[-1] > 0:
        out["D"], out["D_abs"] = lowrank_down(x_hat, L1_bits)
    else:
        out["D"] = np.zeros((x_hat.shape[0], 0), dtype=np.uint16)
        out["D_abs"] = np.zeros((x_hat.shape[0], 0))
    return out


def linear_forward(x_bits: np.ndarray, prep: dict, rows=None) -> dict:
    """Y = bf16(deq(Q(Xhat)) deq(Q(R))^T + D L2 + bias) for the given weight.

    ``prep`` holds inv_lambda, L1 (K x r bf16), L2t (N x r bf16), w_codes,
    w_scales (logical) and bias (or None).  ``rows`` optionally restricts the
    computation to a subset of token rows (for sampled full-size checks).
    Returns dict(Y bf16 bits, Y64 float64 before rounding, plus the act dict).
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    if rows is not None:
        x_bits = x_bits[np.asarray(rows)]
    act = quantize_act(x_bits, prep["inv_lambda"], prep["L1"])
    ax = dequantize(act["x_codes"], act["x_scales"])
    bw = dequantize(prep["w_codes"], prep["w_scales"])
    y = ax @ bw.T
    r = np.asarray(prep["L1"]).shape[-1]
    if r > 0:
        y = y + bf16_to_f64(act["D"]) @ bf16_to_f64(prep["L2t"]).T
    if prep.get("bias") is not None:
        y = y + bf16_to_f64(prep["bias"])[None, :]
    return dict(Y=f64_to_bf16(y), Y64=y, **act)
