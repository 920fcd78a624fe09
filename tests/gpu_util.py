"""Helpers shared by the GPU tests: device buffers from torch, calls through the
C ABI binding, and comparisons with the oracle's tolerances."""
from __future__ import annotations

import numpy as np

from oracle import svdq_ref as ref


def torch():
    import torch as _t
    return _t


def dev_u16(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def dev_f32(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_u8(a: np.ndarray):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def to_np_u16(t) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def empty_u8(n: int):
    t = torch()
    return t.empty(max(int(n), 256), dtype=t.uint8, device="cuda")


def stream() -> int:
    return int(torch().cuda.current_stream().cuda_stream)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 at |x| (8 significant bits), 2^-133 minimum."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.maximum(2.0 ** (e - 7), 2.0 ** -133), 2.0 ** -133)


def check_y(y_gpu_bits: np.ndarray, y_oracle64: np.ndarray, what: str = "Y", y_given_gpu_d=None):
    """Output bar: every element within 4e-3 rms(Y_oracle) plus 2 bf16 ulps of
    itself.  Y_oracle is the oracle's whole forward (its own activation codes,
    scales and D) on the library's exported weight.

    D is a rounding point (bf16 of a K-long sum): the GPU sums in float32 on
    the tensor cores, the oracle in float64, and near a bf16 rounding boundary
    the two round to neighbouring values (D has its own bar, check_d).  When
    `y_given_gpu_d` (the oracle's Y recomputed with the GPU's own D) is given,
    an element beyond the bar against Y_oracle is accepted only if it meets the
    same bar against y_given_gpu_d, i.e. the whole difference is that of D;
    such elements are counted and printed, and may be at most 1 in 10^4.
    Returns max|dY| / rms."""
    yg = ref.bf16_to_f64(y_gpu_bits)
    yo = ref.bf16_to_f64(ref.f64_to_bf16(y_oracle64))
    rms = float(np.sqrt(np.mean(y_oracle64 ** 2)))
    err = np.abs(yg - yo)
    tol = 4e-3 * rms
    bound = tol + 2 * bf16_ulp(yo)
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    over = err > bound
    n_d = 0
    if y_given_gpu_d is not None and np.any(over):
        yd = ref.bf16_to_f64(ref.f64_to_bf16(y_given_gpu_d))
        ok_d = np.abs(yg - yd) <= tol + 2 * bf16_ulp(yd)
        n_d = int((over & ok_d).sum())
        assert n_d <= max(1, err.size // 10000), f"{what}: {n_d} elements differ through D"
        over = over & ~ok_d
    if np.any(over):
        idx = np.argwhere(over)[:5]
        rows = [(int(i), int(j), float(yg[i, j]), float(yo[i, j]), float(err[i, j]),
                 float(bound[i, j])) for i, j in idx]
        raise AssertionError(f"{what}: {int(over.sum())} elements beyond the bound "
                             f"(rms {rms:.3e}); (m, n, gpu, oracle, err, bound): {rows}")
    worst = float(err.max()) if err.size else 0.0
    print(f"{what}: max |dY| / rms = {worst / max(rms, 1e-30):.3e} "
          f"({int((err > 0).sum())} of {err.size} elements differ; "
          f"{n_d} beyond the bar only through the GPU's D)")
    return worst / max(rms, 1e-30)


def y_with_d(y_oracle64: np.ndarray, d_oracle_bits: np.ndarray, d_gpu_bits: np.ndarray,
             L2t_bits: np.ndarray) -> np.ndarray:
    """The oracle's Y with its own low-rank term D L2 replaced by the GPU's D:
    Y - D_o L2 + D_g L2 (float64; the rest of the oracle's sum is unchanged)."""
    L2 = ref.bf16_to_f64(L2t_bits).T
    return y_oracle64 + (ref.bf16_to_f64(d_gpu_bits) - ref.bf16_to_f64(d_oracle_bits)) @ L2


def gpu_d(lin, X_dev, M: int) -> np.ndarray:
    """The activation kernel's D for X (the same kernel, deterministic, that the
    layer's forward runs: svdq_quantize_act_ws), as bf16 bits."""
    import w4a4_rank_corrected_act_b200 as svdq
    t = torch()
    K, r = lin.K, lin.r
    codes = empty_u8(svdq.svdq_act_codes_bytes(M, K))
    scales = empty_u8(svdq.svdq_act_scales_bytes(M, K))
    D = t.empty((M, max(r, 1)), dtype=t.int16, device="cuda")
    nb = svdq.svdq_act_workspace_bytes(M, K, r)
    ws = empty_u8(nb)
    svdq.svdq_quantize_act_ws(X_dev.data_ptr(), M, lin.w, codes.data_ptr(), scales.data_ptr(), D.data_ptr(),
                              ws.data_ptr(), nb, stream())
    t.cuda.synchronize()
    return D.cpu().numpy().view(np.uint16)[:, :r]


def d_propagated_bound(d_oracle_bits: np.ndarray, d_abs: np.ndarray, L2t_bits: np.ndarray):
    """sum_j tol_D[m, j] |L2[j, n]|: how far Y may move when D is within its bar.
    A diagnostic printed beside the Y check, never added to the Y bar."""
    o = ref.bf16_to_f64(d_oracle_bits)
    tol = bf16_ulp(o) + 2.0 ** -14 * d_abs
    return tol @ np.abs(ref.bf16_to_f64(L2t_bits)).T


def check_d(d_gpu_bits: np.ndarray, d_oracle_bits: np.ndarray, d_abs: np.ndarray):
    """D bar: |D_gpu - D_oracle| <= 1 bf16 ulp(D_oracle) + 2^-14 sum_k |Xhat_mk L1_kj|.

    The oracle sums the bf16 x bf16 products in f64 and rounds once; the GPU
    accumulates the same (exact) products in float32: each of 4 partial sums
    takes K/64 tensor-core accumulation steps, each rounding (or truncating) at
    most 2^-23 of a partial bounded by the absolute sum, so the error stays
    below (K/64 + 4) 2^-23 sum|.| <= 2^-14 sum|.| for K <= 16384."""
    g = ref.bf16_to_f64(d_gpu_bits)
    o = ref.bf16_to_f64(d_oracle_bits)
    bound = bf16_ulp(o) + 2.0 ** -14 * d_abs
    err = np.abs(g - o)
    assert np.all(err <= bound), f"D: {int((err > bound).sum())} elements off, max {err.max():.3e}"
