"""ctypes binding of the C ABI in include/svdq.h (argument marshalling only).

Every function here has the name of the C entry point it calls and forwards
plain integers (device / host addresses, sizes, the CUDA stream handle).  No
step of the layer runs in Python: if the shared library is missing or cannot be
loaded, every call raises -- there is no fallback.

`SvdqLinear` is a small convenience owner of one prepared layer whose device
memory comes from PyTorch (PyTorch is used for memory and streams only); its
``format`` is "nvfp4" (default) or "int4".
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libsvdq_b200.so")

SVDQ_OK = 0
SVDQ_FORMAT_NVFP4 = 0
SVDQ_FORMAT_INT4 = 1
FORMAT_NAMES = {"nvfp4": SVDQ_FORMAT_NVFP4, "int4": SVDQ_FORMAT_INT4}
STATUS_NAMES = {
    0: "SVDQ_OK", 1: "SVDQ_ERR_INVALID_ARG", 2: "SVDQ_ERR_UNSUPPORTED_SHAPE",
    3: "SVDQ_ERR_MISALIGNED", 4: "SVDQ_ERR_WORKSPACE_TOO_SMALL", 5: "SVDQ_ERR_CUDA",
    6: "SVDQ_ERR_TIMEOUT", 7: "SVDQ_ERR_SOLVER",
}

# exported symbols, with (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class svdq_weight(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("r", ctypes.c_int32),
        ("has_bias", ctypes.c_int32), ("format", ctypes.c_int32),
        ("w_codes", _P), ("w_scales", _P), ("L1", _P), ("L1f", _P), ("L2t", _P),
        ("inv_lambda", _P), ("bias", _P), ("L1t", _P),
    ]


_WP = ctypes.POINTER(svdq_weight)

SIGNATURES = {
    "svdq_status_string": (ctypes.c_char_p, [_I]),
    "svdq_last_error_detail": (ctypes.c_char_p, []),
    "svdq_version": (ctypes.c_char_p, []),
    "svdq_weight_bytes": (_SZ, [_I, _I, _I, _I]),
    "svdq_act_codes_bytes": (_SZ, [_I, _I]),
    "svdq_act_scales_bytes": (_SZ, [_I, _I]),
    "svdq_forward_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "svdq_prepare_workspace_bytes": (_SZ, [_I, _I, _I]),
    "svdq_weight_bind": (_I, [_P, _SZ, _I, _I, _I, _I, _WP]),
    "svdq_weight_bind_format": (_I, [_P, _SZ, _I, _I, _I, _I, _I, _WP]),
    "svdq_prepare_weight": (_I, [_P, _P, _P, _WP, _P, _SZ, _P]),
    "svdq_quantize_act": (_I, [_P, _I, _WP, _P, _P, _P, _P]),
    "svdq_act_workspace_bytes": (_SZ, [_I, _I, _I]),
    "svdq_quantize_act_ws": (_I, [_P, _I, _WP, _P, _P, _P, _P, _SZ, _P]),
    "svdq_gemm": (_I, [_P, _P, _P, _I, _WP, _P, _P]),
    "svdq_linear_forward": (_I, [_P, _I, _WP, _P, _P, _SZ, _P]),
    "svdq_linear_forward_host": (_I, [_P, _I, _WP, _P, _P, _P, _P, _SZ, _P]),
    "svdq_linear_forward_noalloc": (_I, [_P, _I, _WP, _P, _P]),
    "svdq_gemm_heads": (_I, [_P, _P, _P, _I, _WP, _I, _P, _P]),
    "svdq_linear_forward_heads": (_I, [_P, _I, _WP, _I, _P, _P, _SZ, _P]),
    "svdq_mlp_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "svdq_mlp_forward": (_I, [_P, _I, _WP, _WP, _P, _P, _P, _SZ, _P]),
    "svdq_weight_export": (_I, [_WP, _P, _P, _P, _P, _P, _P]),
    "svdq_weight_import": (_I, [_WP, _P, _P, _P, _P, _P, _P, _P]),
    "svdq_calib_absmax": (_I, [_P, _I, _I, _P, _P]),
    "svdq_calibrate_lambda": (_I, [_P, _P, _I, _I, ctypes.c_float, _P, _P]),
    "svdq_scales_to_logical": (_I, [_P, _I, _I, _P]),
    "svdq_scales_to_native": (_I, [_P, _I, _I, _P]),
    "svdq_act_scales_to_logical": (_I, [_P, _I, _I, _P]),
    "svdq_int4_scales_to_logical": (_I, [_P, _I, _I, _I, _P]),
    "svdq_int4_scales_to_native": (_I, [_P, _I, _I, _I, _P]),
    "svdq_set_override": (_I, [_I, _I]),
    "svdq_get_device_status": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "svdq_clear_device_status": (_I, [_P]),
    "svdq_selftest_wait_timeout": (_I, [ctypes.c_uint64, _P]),
    "svdq_selftest_quotient": (_I, [ctypes.POINTER(ctypes.c_uint64)]),
    "svdq_selftest_conversions": (_I, [ctypes.POINTER(ctypes.c_uint64)]),
}

_lib: Optional[ctypes.CDLL] = None


class SvdqError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        msg = f"{fn} -> {STATUS_NAMES.get(status, status)}"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """Load libsvdq_b200.so (built by ``w4a4_rank_corrected_act_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m w4a4_rank_corrected_act_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(handle, name)
            f.restype = res
            f.argtypes = args
        _lib = handle
    return _lib


def _check(fn: str, status: int) -> None:
    if status != SVDQ_OK:
        detail = lib().svdq_last_error_detail().decode(errors="replace")
        raise SvdqError(fn, status, detail if status in (5, 7) else "")


def _call(fn: str, *args) -> None:
    _check(fn, getattr(lib(), fn)(*args))


# --------------------------------------------------------------------------
# one wrapper per entry point (same names as the C ABI)
# --------------------------------------------------------------------------

def svdq_status_string(s: int) -> str:
    return lib().svdq_status_string(s).decode()


def svdq_version() -> str:
    return lib().svdq_version().decode()


def svdq_weight_bytes(N: int, K: int, r: int, has_bias: int) -> int:
    return lib().svdq_weight_bytes(N, K, r, has_bias)


def svdq_act_codes_bytes(M: int, K: int) -> int:
    return lib().svdq_act_codes_bytes(M, K)


def svdq_act_scales_bytes(M: int, K: int) -> int:
    return lib().svdq_act_scales_bytes(M, K)


def svdq_forward_workspace_bytes(M: int, N: int, K: int, r: int) -> int:
    return lib().svdq_forward_workspace_bytes(M, N, K, r)


def svdq_prepare_workspace_bytes(N: int, K: int, r: int) -> int:
    return lib().svdq_prepare_workspace_bytes(N, K, r)


def svdq_weight_bind(buf: int, nbytes: int, N: int, K: int, r: int, has_bias: int) -> svdq_weight:
    w = svdq_weight()
    _call("svdq_weight_bind", buf, nbytes, N, K, r, has_bias, ctypes.byref(w))
    return w


def svdq_weight_bind_format(buf: int, nbytes: int, N: int, K: int, r: int, has_bias: int,
                            format: int) -> svdq_weight:
    w = svdq_weight()
    _call("svdq_weight_bind_format", buf, nbytes, N, K, r, has_bias, format, ctypes.byref(w))
    return w


def svdq_prepare_weight(W: int, lam: int, bias: int, w: svdq_weight, ws: int, ws_bytes: int,
                        stream: int) -> None:
    _call("svdq_prepare_weight", W, lam, bias or None, ctypes.byref(w), ws, ws_bytes, stream or None)


def svdq_quantize_act(X: int, M: int, w: svdq_weight, x_codes: int, x_scales: int, D: int,
                      stream: int) -> None:
    _call("svdq_quantize_act", X, M, ctypes.byref(w), x_codes, x_scales, D or None, stream or None)


def svdq_act_workspace_bytes(M: int, K: int, r: int) -> int:
    return int(lib().svdq_act_workspace_bytes(M, K, r))


def svdq_quantize_act_ws(X: int, M: int, w: svdq_weight, x_codes: int, x_scales: int, D: int, ws: int,
                         ws_bytes: int, stream: int) -> None:
    """The forward's own activation kernel (128-row CTAs, D on the tensor cores)."""
    _call("svdq_quantize_act_ws", X, M, ctypes.byref(w), x_codes, x_scales, D or None, ws, ws_bytes,
          stream or None)


def svdq_gemm(x_codes: int, x_scales: int, D: int, M: int, w: svdq_weight, Y: int,
              stream: int) -> None:
    _call("svdq_gemm", x_codes, x_scales, D or None, M, ctypes.byref(w), Y, stream or None)


def svdq_linear_forward(X: int, M: int, w: svdq_weight, Y: int, ws: int, ws_bytes: int,
                        stream: int) -> None:
    _call("svdq_linear_forward", X, M, ctypes.byref(w), Y, ws, ws_bytes, stream or None)


def svdq_gemm_heads(x_codes: int, x_scales: int, D: int, M: int, w: svdq_weight, head_dim: int,
                    Y: int, stream: int) -> None:
    _call("svdq_gemm_heads", x_codes, x_scales, D or None, M, ctypes.byref(w), head_dim, Y, stream or None)


def svdq_linear_forward_heads(X: int, M: int, w: svdq_weight, head_dim: int, Y: int, ws: int,
                              ws_bytes: int, stream: int) -> None:
    _call("svdq_linear_forward_heads", X, M, ctypes.byref(w), head_dim, Y, ws, ws_bytes, stream or None)


def svdq_linear_forward_host(X_host: int, M: int, w: svdq_weight, Y_host: int, X_dev: int,
                             Y_dev: int, ws: int, ws_bytes: int, stream: int) -> None:
    _call("svdq_linear_forward_host", X_host, M, ctypes.byref(w), Y_host, X_dev, Y_dev, ws,
          ws_bytes, stream or None)


def svdq_linear_forward_noalloc(X: int, M: int, w: svdq_weight, Y: int, stream: int) -> None:
    """Whole layer with the library's fixed device scratch (no allocation);
    for callers that cannot allocate device memory or pass a workspace."""
    st = lib().svdq_linear_forward_noalloc(X, M, ctypes.byref(w), Y, stream or None)
    if st == 4:   # shape too large for the fixed scratch: the library says by how much
        raise SvdqError("svdq_linear_forward_noalloc", st,
                        lib().svdq_last_error_detail().decode(errors="replace"))
    _check("svdq_linear_forward_noalloc", st)


def svdq_mlp_workspace_bytes(M: int, K: int, F: int, N: int, r_up: int, r_down: int) -> int:
    return int(lib().svdq_mlp_workspace_bytes(M, K, F, N, r_up, r_down))


def svdq_mlp_forward(X: int, M: int, up: svdq_weight, down: svdq_weight, Y: int, H_out: int, ws: int,
                     ws_bytes: int, stream: int) -> None:
    """MLP pair (up-projection, GELU, down-projection) with the GELU and the
    down-projection's activation quantisation in the up-projection's epilogue."""
    _call("svdq_mlp_forward", X or None, M, ctypes.byref(up), ctypes.byref(down), Y or None, H_out or None,
          ws or None, ws_bytes, stream or None)


def svdq_weight_export(w: svdq_weight, host_codes: int, host_scales: int, host_L1: int,
                       host_L2t: int, host_inv_lambda: int, stream: int) -> None:
    _call("svdq_weight_export", ctypes.byref(w), host_codes or None, host_scales or None,
          host_L1 or None, host_L2t or None, host_inv_lambda or None, stream or None)


def svdq_weight_import(w: svdq_weight, host_codes: int, host_scales: int, host_L1: int,
                       host_L2t: int, host_inv_lambda: int, host_bias: int, stream: int) -> None:
    _call("svdq_weight_import", ctypes.byref(w), host_codes, host_scales, host_L1 or None,
          host_L2t or None, host_inv_lambda, host_bias or None, stream or None)


def svdq_calib_absmax(A: int, rows: int, K: int, colmax: int, stream: int) -> None:
    _call("svdq_calib_absmax", A, rows, K, colmax, stream or None)


def svdq_calibrate_lambda(x_absmax: int, W: int, N: int, K: int, alpha: float, lam: int,
                          stream: int) -> None:
    _call("svdq_calibrate_lambda", x_absmax, W, N, K, float(alpha), lam, stream or None)


def svdq_scales_to_logical(native: int, rows: int, K: int, logical: int) -> None:
    _call("svdq_scales_to_logical", native, rows, K, logical)


def svdq_act_scales_to_logical(native: int, M: int, K: int, logical: int) -> None:
    _call("svdq_act_scales_to_logical", native, M, K, logical)


def svdq_scales_to_native(logical: int, rows: int, K: int, native: int) -> None:
    _call("svdq_scales_to_native", logical, rows, K, native)


def svdq_int4_scales_to_logical(native: int, rows: int, rows_pad: int, K: int, logical: int) -> None:
    _call("svdq_int4_scales_to_logical", native, rows, rows_pad, K, logical)


def svdq_int4_scales_to_native(logical: int, rows: int, rows_pad: int, K: int, native: int) -> None:
    _call("svdq_int4_scales_to_native", logical, rows, rows_pad, K, native)


SVDQ_OVERRIDE_ACT_KSPLIT = 1
SVDQ_OVERRIDE_GEMM_BN = 2
SVDQ_OVERRIDE_HOST_CHUNK_ROWS = 3
SVDQ_OVERRIDE_SMALL_M = 4
SVDQ_OVERRIDE_ACT_KERNEL = 5


def svdq_set_override(which: int, value: int) -> None:
    _call("svdq_set_override", which, value)


class override:
    """Context manager: set one launch-choice override, restore automatic (0) on exit."""

    def __init__(self, which: int, value: int):
        self.which, self.value = which, value

    def __enter__(self):
        svdq_set_override(self.which, self.value)
        return self

    def __exit__(self, *exc):
        svdq_set_override(self.which, 0)
        return False


def svdq_get_device_status(stream: int = 0) -> int:
    """Returns the raw device status word (0 = no kernel gave up a wait)."""
    detail = ctypes.c_uint32(0)
    st = lib().svdq_get_device_status(stream or None, ctypes.byref(detail))
    if st not in (SVDQ_OK, 6):
        _check("svdq_get_device_status", st)
    return int(detail.value)


def svdq_clear_device_status(stream: int = 0) -> None:
    _call("svdq_clear_device_status", stream or None)


def svdq_selftest_wait_timeout(limit_ns: int, stream: int = 0) -> None:
    _call("svdq_selftest_wait_timeout", int(limit_ns), stream or None)


def svdq_selftest_quotient() -> tuple:
    """(normal-range quotient mismatches, code mismatches, subnormal-range
    quotient mismatches) of the activation quantiser's division-free path over
    its exhaustive sweep; the first two are 0 on a correct build."""
    out = (ctypes.c_uint64 * 3)()
    _call("svdq_selftest_quotient", out)
    return int(out[0]), int(out[1]), int(out[2])


def svdq_selftest_conversions() -> tuple:
    """(E4M3, E2M1, bf16) mismatch counts of the device conversions over every
    non-negative finite float32; all 0 on a correct device."""
    out = (ctypes.c_uint64 * 3)()
    _call("svdq_selftest_conversions", out)
    return int(out[0]), int(out[1]), int(out[2])


# --------------------------------------------------------------------------
# convenience owner of one prepared layer (device memory from torch)
# --------------------------------------------------------------------------

def _stream_handle(stream=None) -> int:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


# weight-file format tags written by SvdqLinear.save
_FILE_FORMATS = {"nvfp4": "svdq-w4a4-nvfp4-1", "int4": "svdq-w4a4-int4-1"}


class SvdqLinear:
    """A prepared SVDQuant W4A4 linear on the current CUDA device.

    ``W`` (N x K), ``lam`` (K, float32) and ``bias`` (N or None) are device
    tensors; the weight is prepared once with ``svdq_prepare_weight`` and kept
    in one torch-allocated buffer bound with ``svdq_weight_bind_format``.
    ``format`` is "nvfp4" (the Blackwell format, default) or "int4".
    """

    def __init__(self, W, lam, bias=None, r: int = 32, stream=None, format: str = "nvfp4"):
        import torch
        N, K = W.shape
        self._bind(int(N), int(K), int(r), bias is not None, W.device, format)
        ws_bytes = svdq_prepare_workspace_bytes(self.N, self.K, self.r)
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=W.device)
        Wc = W.contiguous()
        lc = lam.contiguous()
        bc = bias.contiguous() if bias is not None else None
        svdq_prepare_weight(Wc.data_ptr(), lc.data_ptr(), bc.data_ptr() if bc is not None else 0,
                            self.w, ws.data_ptr(), ws_bytes, _stream_handle(stream))
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
        del ws

    def _bind(self, N: int, K: int, r: int, has_bias: bool, device, format: str = "nvfp4") -> None:
        import torch
        if format not in FORMAT_NAMES:
            raise ValueError(f"format must be one of {sorted(FORMAT_NAMES)}")
        self.N, self.K, self.r = N, K, r
        self.has_bias = has_bias
        self.format = format
        nbytes = svdq_weight_bytes(self.N, self.K, self.r, int(self.has_bias))
        if nbytes == 0:
            raise SvdqError("svdq_weight_bytes", 2, f"N={N} K={K} r={r}")
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.w = svdq_weight_bind_format(self.buf.data_ptr(), nbytes, self.N, self.K, self.r,
                                         int(self.has_bias), FORMAT_NAMES[format])

    @classmethod
    def from_export(cls, exp: dict, bias=None, device="cuda", stream=None, format: Optional[str] = None):
        """A layer from host arrays in the layouts of ``export()`` (bias: N uint16
        bf16 bits or None), loaded with ``svdq_weight_import``.  ``format`` defaults
        to the one the scales imply: fp16 group scales (uint16) are INT4, E4M3
        codes (uint8) NVFP4."""
        import numpy as np
        if format is None:
            format = "int4" if np.asarray(exp["w_scales"]).dtype == np.uint16 else "nvfp4"
        self = cls.__new__(cls)
        N, K2 = exp["w_codes"].shape
        r = int(exp["L1"].shape[1]) if exp.get("L1") is not None else 0
        self._bind(int(N), int(K2) * 2, r, bias is not None, device, format)
        # every host array stays referenced until the (synchronous) import returns
        codes = np.ascontiguousarray(exp["w_codes"], dtype=np.uint8)
        scales = np.ascontiguousarray(exp["w_scales"], dtype=np.uint16 if format == "int4" else np.uint8)
        L1 = np.ascontiguousarray(exp["L1"], dtype=np.uint16) if r else None
        L2t = np.ascontiguousarray(exp["L2t"], dtype=np.uint16) if r else None
        inv = np.ascontiguousarray(exp["inv_lambda"], dtype=np.float32)
        b = np.ascontiguousarray(bias, dtype=np.uint16) if bias is not None else None
        svdq_weight_import(self.w, codes.ctypes.data, scales.ctypes.data,
                           L1.ctypes.data if r else 0, L2t.ctypes.data if r else 0, inv.ctypes.data,
                           b.ctypes.data if b is not None else 0, _stream_handle(stream))
        return self

    def bias_host(self):
        """The layer's bias as uint16 bf16 bits (numpy), or None."""
        if not self.has_bias:
            return None
        off = self.w.bias - self.buf.data_ptr()
        return self.buf[off:off + 2 * self.N].cpu().numpy().view("uint16").copy()

    def save(self, path) -> None:
        """Write the prepared weight (logical layouts, bias included) to an .npz file."""
        import numpy as np
        exp = self.export()
        extra = {"bias": self.bias_host()} if self.has_bias else {}
        np.savez(path, format=np.array(_FILE_FORMATS[self.format]), N=self.N, K=self.K, r=self.r, **exp, **extra)

    @classmethod
    def load(cls, path, device="cuda", stream=None):
        """A layer from a file written by ``save``."""
        import numpy as np
        with np.load(path) as z:
            fmt = {v: k for k, v in _FILE_FORMATS.items()}.get(str(z["format"]))
            if fmt is None:
                raise ValueError(f"{path}: not an SVDQuant weight file")
            exp = {k: z[k] for k in ("w_codes", "w_scales", "L1", "L2t", "inv_lambda")}
            bias = z["bias"] if "bias" in z.files else None
        return cls.from_export(exp, bias=bias, device=device, stream=stream, format=fmt)

    def workspace_bytes(self, M: int) -> int:
        return svdq_forward_workspace_bytes(M, self.N, self.K, self.r)

    def forward(self, X, Y=None, ws=None, stream=None):
        import torch
        M = X.shape[0]
        if Y is None:
            Y = torch.empty((M, self.N), dtype=torch.bfloat16, device=X.device)
        nb = self.workspace_bytes(M)
        if ws is None:
            ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=X.device)
        svdq_linear_forward(X.data_ptr(), M, self.w, Y.data_ptr(), ws.data_ptr(), nb,
                            _stream_handle(stream))
        return Y

    def export(self):
        """Host copies of the prepared weight in logical layouts (numpy arrays)."""
        import numpy as np
        codes = np.empty((self.N, self.K // 2), np.uint8)
        if self.format == "int4":
            scales = np.empty((self.N, self.K // 64), np.uint16)     # fp16 bits
        else:
            scales = np.empty((self.N, self.K // 16), np.uint8)      # E4M3 codes
        L1 = np.empty((self.K, self.r), np.uint16)
        L2t = np.empty((self.N, self.r), np.uint16)
        inv = np.empty(self.K, np.float32)
        svdq_weight_export(self.w, codes.ctypes.data, scales.ctypes.data,
                           L1.ctypes.data if self.r else 0, L2t.ctypes.data if self.r else 0,
                           inv.ctypes.data, _stream_handle())
        return dict(w_codes=codes, w_scales=scales, L1=L1, L2t=L2t, inv_lambda=inv)


def calibrate_lambda(W, X_batches, alpha: float = 0.5, stream=None):
    """Smoothing factors for the weight W (N x K bf16, device) from calibration
    activations (an iterable of M_i x K bf16 device tensors): the column
    maxima of |X| over all batches (svdq_calib_absmax), then
    svdq_calibrate_lambda with migration strength alpha.  Returns a device
    float32 tensor of K entries, the ``lam`` input of SvdqLinear."""
    import torch
    N, K = W.shape
    sh = _stream_handle(stream)
    colmax = torch.zeros(K, dtype=torch.float32, device=W.device)
    for X in X_batches:
        Xc = X.contiguous()
        svdq_calib_absmax(Xc.data_ptr(), int(Xc.shape[0]), int(K), colmax.data_ptr(), sh)
    lam = torch.empty(K, dtype=torch.float32, device=W.device)
    Wc = W.contiguous()
    svdq_calibrate_lambda(colmax.data_ptr(), Wc.data_ptr(), int(N), int(K), alpha, lam.data_ptr(), sh)
    return lam
