"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module is shared by the CPU oracle, the CUDA path's tests and the
benchmark.  It holds *no* arithmetic of the method itself (no smoothing, no
SVD, no quantisation): it only draws random matrices with the shapes and
statistics of diffusion-transformer linears and rounds them to bf16.

The five workloads follow the configuration list that accompanies the
method description (single small linear; DiT QKV projection at 1024x1024;
DiT MLP up/down pair; small-M adaLN projection; all four linears of one
3072-hidden DiT block).  The pages themselves only benchmark end-to-end image
generation with trained FLUX/ERNIE checkpoints (aiphreaks.com "Bringing
Nunchaku 4-bit Diffusion Inference to Diffusers", section "Technical
Breakdown and Performance Metrics"; chaosnode.de "Nunchaku Lite",
section "Praxisbeispiel"), which are not available here: these synthetic,
DiT-shaped inputs stand in for them.

Draw order inside one linear (fixed, so every consumer sees the same arrays):
X base, outlier-channel indices, W base, W structure, bias.

The smoothing factor lambda is an *input* of the layer (the caller calibrates
it); the recipe used for every workload is
    lambda_k = sqrt(max_m |X_mk| / max_n |W_nk|),   lambda_k = 1 if either max is 0,
computed in float64 from the bf16 values and rounded to float32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "LinearSpec", "WORKLOADS", "workload", "make_linear", "to_bf16_bits",
    "bf16_bits_to_f32", "calibrate_lambda", "gelu_tanh",
]


@dataclasses.dataclass(frozen=True)
class LinearSpec:
    """Shape and input recipe of one synthetic linear layer Y = X W^T + b."""
    name: str
    M: int
    K: int
    N: int
    r: int
    seed: object                  # int, or a tuple for the linears of a block
    x_kind: str = "normal"        # "normal" | "gelu"
    x_outliers: int = 4           # number of outlier input channels
    x_outlier_scale: float = 40.0
    w_kind: str = "plain"         # "plain" | "cols" | "spike"
    w_cols: int = 2               # outlier input columns of W ("cols")
    w_col_scale: float = 10.0
    spike_rank: int = 8           # "spike": number of unit singular directions
    spike_value: float = 5.0      # "spike": singular value of each direction

    @property
    def flops(self) -> int:
        """Dense 4-bit GEMM flops 2*M*N*K (the low-rank branch is not counted)."""
        return 2 * self.M * self.N * self.K

    @property
    def lowrank_flops(self) -> int:
        return 2 * self.M * self.r * (self.K + self.N)


def _cfg2_x(K: int) -> dict:
    # 1% of channels scaled x50 (heavy-tail outliers)
    return dict(x_kind="normal", x_outliers=int(round(0.01 * K)), x_outlier_scale=50.0)


def _block(M: int, tag: str) -> List[LinearSpec]:
    shapes = [("qkv", 3072, 9216), ("out", 3072, 3072), ("up", 3072, 12288), ("down", 12288, 3072)]
    out = []
    for i, (nm, K, N) in enumerate(shapes):
        out.append(LinearSpec(f"{tag}_{nm}", M, K, N, 32, (4, i), **_cfg2_x(K),
                              w_kind="spike"))
    return out


WORKLOADS: Dict[str, LinearSpec] = {}
for _s in [
    # 1: single small linear (the case the oracle finishes in seconds)
    LinearSpec("small", 256, 512, 512, 32, 0, x_outliers=4, x_outlier_scale=40.0,
               w_kind="cols", w_cols=2, w_col_scale=10.0),
    # 2: DiT joint-attention QKV projection at 1024x1024 (4096 image + 512 text tokens)
    LinearSpec("qkv", 4608, 3072, 9216, 32, 1, **_cfg2_x(3072), w_kind="spike"),
    # 3: DiT MLP pair
    LinearSpec("mlp_up", 4608, 3072, 12288, 32, 2, **_cfg2_x(3072), w_kind="cols"),
    LinearSpec("mlp_down", 4608, 12288, 3072, 32, 2, x_kind="gelu",
               x_outliers=int(round(0.005 * 12288)), x_outlier_scale=30.0, w_kind="cols"),
    # 4: small-M bandwidth case (adaLN modulation / low-res preview)
    LinearSpec("small_m", 16, 3072, 18432, 32, 3, x_outliers=4, x_outlier_scale=40.0,
               w_kind="plain"),
] + _block(4608, "block_b1") + _block(18432, "block_b4"):
    WORKLOADS[_s.name] = _s


def workload(name: str) -> LinearSpec:
    return WORKLOADS[name]


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    """tanh-approximated GELU, used only to shape the down-projection input."""
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def calibrate_lambda(x_bits: np.ndarray, w_bits: np.ndarray) -> np.ndarray:
    """Per-input-channel smoothing factor (input recipe, see module docstring)."""
    xm = np.abs(bf16_bits_to_f32(x_bits).astype(np.float64)).max(axis=0)
    wm = np.abs(bf16_bits_to_f32(w_bits).astype(np.float64)).max(axis=0)
    lam = np.ones_like(xm)
    ok = (xm > 0) & (wm > 0)
    lam[ok] = np.sqrt(xm[ok] / wm[ok])
    return lam.astype(np.float32)


def _orthonormal(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return q


def make_linear(spec: LinearSpec, M: Optional[int] = None) -> dict:
    """Draw one linear's inputs.

    Returns a dict with uint16 bf16 bit arrays ``X`` (M x K), ``W`` (N x K),
    ``bias`` (N) and the float32 calibration vector ``lam`` (K).  ``M``
    overrides the token count (the rows are a prefix of a larger draw only when
    the override equals spec.M; it is meant for reduced-size variants).
    """
    M = spec.M if M is None else int(M)
    K, N = spec.K, spec.N
    seed = spec.seed if isinstance(spec.seed, int) else list(spec.seed)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    if spec.x_kind == "gelu":
        x = gelu_tanh(x)
    if spec.x_outliers > 0:
        idx = rng.choice(K, size=min(spec.x_outliers, K), replace=False)
        x[:, idx] *= spec.x_outlier_scale
    w = rng.standard_normal((N, K)) * 0.02
    if spec.w_kind == "cols":
        cols = rng.choice(K, size=min(spec.w_cols, K), replace=False)
        w[:, cols] *= spec.w_col_scale
    elif spec.w_kind == "spike":
        k = min(spec.spike_rank, N, K)
        u = _orthonormal(rng, N, k)
        v = _orthonormal(rng, K, k)
        w += spec.spike_value * (u @ v.T)
    elif spec.w_kind != "plain":
        raise ValueError(spec.w_kind)
    bias = rng.standard_normal(N) * 0.01
    X = to_bf16_bits(x)
    W = to_bf16_bits(w)
    B = to_bf16_bits(bias)
    return dict(X=X, W=W, bias=B, lam=calibrate_lambda(X, W), spec=spec, M=M)


def random_bf16(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """Small helper for ad-hoc test shapes: N(0, scale^2) rounded to bf16 bits."""
    return to_bf16_bits(rng.standard_normal(shape) * scale)
