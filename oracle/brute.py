"""Brute-force twin of the oracle for tiny shapes (TEST INFRASTRUCTURE ONLY).

Independent restatement of the layer with explicit Python loops over scalars:
no NumPy matmul, no table search.  Conversions are written in closed form from
the format definitions (E2M1: 1 sign, 2 exponent, 1 mantissa bit, values
{0, .5, 1, 1.5, 2, 3, 4, 6}; E4M3: 4 exponent bits with bias 7, 3 mantissa
bits, subnormal step 2^-9, largest finite 448; bf16: 8 significant bits) with
Python's round(), which rounds half to even.  Float32 operations are done on
np.float32 scalars (IEEE single, round to nearest even).

It follows the same readings R1-R9 as ``oracle/svdq_ref.py`` (see there), and
for the INT4 variant R15-R18 of ``oracle/int4_ref.py``, where half precision
is rounded with Python's own binary16 packing (struct format "e", round half
to even) instead of NumPy's.  It takes L1/L2 as given: the SVD itself is
pinned by the textbook identities in the tests, not re-derived here.
"""
from __future__ import annotations

import math
import struct

import numpy as np

F32 = np.float32


def bf16_round(x: float) -> float:
    """Round a float64 value to the nearest bf16 value (ties to even)."""
    if x == 0.0 or not math.isfinite(x):
        return x
    m, e = math.frexp(x)                    # x = m * 2^e, 0.5 <= |m| < 1
    if e - 1 < -126:                        # bf16 subnormal: multiples of 2^-133
        return round(x * 2.0 ** 133) * 2.0 ** -133
    return math.ldexp(round(m * 256.0), e - 8)


def e2m1_round(q: float) -> float:
    """Nearest E2M1 magnitude-with-sign (ties to even code), saturating at 6."""
    a = abs(q)
    if a < 2.0:
        step = 0.5
    elif a < 4.0:
        step = 1.0
    else:
        step = 2.0
    v = step * round(a / step)
    v = min(v, 6.0)
    return math.copysign(v, q)


_E2M1_CODE = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def e2m1_code(v: float) -> int:
    c = _E2M1_CODE[abs(v)]
    return c | (8 if math.copysign(1.0, v) < 0 else 0)


def e4m3_round(x: float) -> float:
    """Nearest non-negative E4M3 value (ties to even), saturating at 448."""
    if x <= 0.0:
        return 0.0
    if x < 2.0 ** -6:
        step = 2.0 ** -9
    else:
        _, e = math.frexp(x)
        step = 2.0 ** (e - 1 - 3)
    v = step * round(x / step)
    return min(v, 448.0)


def e4m3_code(v: float) -> int:
    if v < 2.0 ** -6:
        return int(v / 2.0 ** -9)
    _, e = math.frexp(v)
    E = e - 1
    m = int(round((v / 2.0 ** E - 1.0) * 8))
    return ((E + 7) << 3) | m


def quantize_row(vals):
    """One row of float32 values -> (list of 4-bit codes, list of scale codes)."""
    K = len(vals)
    codes, scodes = [], []
    for b in range(K // 16):
        blk = [F32(vals[b * 16 + i]) for i in range(16)]
        a = F32(0)
        for v in blk:
            a = max(a, F32(abs(v)))
        s = e4m3_round(float(F32(a) / F32(6)))
        scodes.append(e4m3_code(s))
        for v in blk:
            if s == 0.0:
                q = math.copysign(0.0, float(v))
            else:
                q = float(F32(v) / F32(s))
            codes.append(e2m1_code(e2m1_round(q)))
    return codes, scodes


def code_value(c: int) -> float:
    mag = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0][c & 7]
    return -mag if c & 8 else mag


def e4m3_value(c: int) -> float:
    e, m = (c >> 3) & 15, c & 7
    return (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)


def _bf(bits) -> float:
    return float(np.array([int(bits) << 16], dtype=np.uint32).view(np.float32)[0])


def f16_round(x: float) -> float:
    """Nearest binary16 value of a non-negative float (ties to even), saturating
    at 65504, by Python's struct packing."""
    return struct.unpack("<e", struct.pack("<e", min(x, 65504.0)))[0]


def quantize_row_int4(vals):
    """One row of float32 values -> (list of int codes in [-8, 7], list of fp16 scale values)."""
    K = len(vals)
    codes, scales = [], []
    for g in range(K // 64):
        grp = [F32(vals[g * 64 + i]) for i in range(64)]
        a = F32(0)
        for v in grp:
            a = max(a, F32(abs(v)))
        s = f16_round(float(F32(a) / F32(7)))
        scales.append(s)
        for v in grp:
            if s == 0.0:
                codes.append(0)
            else:
                q = round(float(F32(v) / F32(s)))     # half to even
                codes.append(max(-8, min(7, q)))
    return codes, scales


def _forward(X_bits, W_bits, lam, bias_bits, L1_bits, L2_bits, quantize, deq_x):
    M, K = len(X_bits), len(X_bits[0])
    N = len(W_bits)
    r = len(L1_bits[0]) if K and len(L1_bits) else 0
    inv = [F32(1) / F32(lam[k]) for k in range(K)]
    # activation side
    xhat = [[F32(F32(_bf(X_bits[m][k])) * inv[k]) for k in range(K)] for m in range(M)]
    xq = [quantize(row) for row in xhat]
    # low-rank down projection, f64 sum of bf16 x bf16 products
    L1 = [[_bf(L1_bits[k][j]) for j in range(r)] for k in range(K)]
    L2 = [[_bf(L2_bits[j][n]) for n in range(N)] for j in range(r)]
    D = []
    for m in range(M):
        row = []
        for j in range(r):
            acc = 0.0
            for k in range(K):
                acc += bf16_round(float(xhat[m][k])) * L1[k][j]
            row.append(bf16_round(acc))
        D.append(row)
    # weight side: smoothing, residual (f64, increasing j), quantisation
    wq = []
    for n in range(N):
        rrow = []
        for k in range(K):
            what = F32(F32(_bf(W_bits[n][k])) * F32(lam[k]))
            acc = 0.0
            for j in range(r):
                acc += L1[k][j] * L2[j][n]
            rrow.append(F32(float(what) - acc))
        wq.append(quantize(rrow))
    # output in float64
    Y = []
    for m in range(M):
        yrow = []
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += deq_x(xq[m], k) * deq_x(wq[n], k)
            for j in range(r):
                acc += D[m][j] * L2[j][n]
            if bias_bits is not None:
                acc += _bf(bias_bits[n])
            yrow.append(acc)
        Y.append(yrow)
    return dict(x_codes=[q[0] for q in xq], x_scales=[q[1] for q in xq],
                w_codes=[q[0] for q in wq], w_scales=[q[1] for q in wq], D=D, Y64=Y)


def forward(X_bits, W_bits, lam, bias_bits, L1_bits, L2_bits):
    """Whole NVFP4 layer on tiny inputs with explicit loops.

    X_bits M x K, W_bits N x K (bf16 bits), lam K (float32), bias_bits N or None,
    L1_bits K x r, L2_bits r x N (bf16 bits).  Returns a dict with unpacked x/w
    codes, x/w scale codes, D (bf16 values, M x r) and Y64 (float64, M x N).
    """
    return _forward(X_bits, W_bits, lam, bias_bits, L1_bits, L2_bits, quantize_row,
                    lambda q, k: code_value(q[0][k]) * e4m3_value(q[1][k // 16]))


def forward_int4(X_bits, W_bits, lam, bias_bits, L1_bits, L2_bits):
    """Whole INT4 layer on tiny inputs (K a multiple of 64) with explicit loops;
    same arguments and result fields as forward(), the codes as signed ints and
    the scales as fp16 values."""
    return _forward(X_bits, W_bits, lam, bias_bits, L1_bits, L2_bits, quantize_row_int4,
                    lambda q, k: q[0][k] * q[1][k // 64])
