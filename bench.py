#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload qkv]

One step = one ``svdq_linear_forward`` (activation kernel + block-scaled FP4
GEMM with the fused low-rank branch and bias) over the DiT joint-attention QKV
projection at 1024x1024 (M = 4608 tokens, K = 3072, N = 9216, r = 32), inputs
resident in HBM.  L2 is flushed (a 256 MiB write, outside the per-step CUDA
events) between steps.  Metric: TFLOP/s = 2 M N K / device time per step
(the low-rank flops 2 M r (K + N) are not counted).

Multi-GPU (torchrun, one rank per GPU): the layer is run as independent
replicas (token-parallel data parallelism, weights replicated, no collective on
the data path); value = all ranks' flops / max-over-ranks device time.

``--format int4`` runs the same step with the layer's INT4 variant (signed
4-bit codes, fp16 scale per 64 elements; integer group sums on the 8-bit
integer warp MMA) and reports it against the 8-bit integer tensor peak.

``--impl reference`` times the CPU oracle (the only other implementation of the
method available) on the host cores, on a bounded row sample of the same
workload, and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SVDQ W4A4 linear TFLOP/s and % of B200 FP4 tensor peak (HBM % at small M)"
UNIT = "TFLOP/s"
FP4_SPEC_TFLOPS = 9000.0          # dense NVFP4, NVIDIA B200 datasheet
HBM_SPEC_GBS = 8000.0             # HBM3e, NVIDIA B200 datasheet (DGX figure)
FP4_OVER_BF16 = 4.0               # nominal dense ratio fp4 : bf16 (9 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = os.path.join(ROOT, "w4a4_rank_corrected_act_b200", "csrc")
# the sources each kernel is compiled from (a profile is stale once any changed)
GEMM_SRC = [os.path.join(_CSRC, f) for f in ("fp4_gemm.cuh", "ptx.cuh", "nvfp4.cuh")]
ACT_SRC = [os.path.join(_CSRC, f) for f in ("act_quant.cuh", "ptx.cuh", "nvfp4.cuh")]
INT4_SRC = [os.path.join(_CSRC, f) for f in ("int4.cuh", "act_quant.cuh", "ptx.cuh", "nvfp4.cuh")]
A128_SRC = [os.path.join(_CSRC, f) for f in ("act128.cuh", "ptx.cuh", "nvfp4.cuh")]
I8_OVER_BF16 = 2.0                # nominal dense ratio int8 : bf16 (4.5 / 2.25 POPS)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def _of_sustained(value):
    """value / (4 x the measured sustained bf16 throughput), or None without it."""
    sus = _peaks()[0].get("bf16_tflops_sustained")
    return round(value / (sus * FP4_OVER_BF16), 4) if sus else None


def _src_sha(paths) -> str:
    h = hashlib.sha256()
    for path in paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _profile_traffic(kernel_src: str, name: str):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (sha recorded in the summary); else None."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    sha = _src_sha(kernel_src)
    traffic, src = None, None
    with open(p) as f:
        for line in f:
            if line.startswith("source_sha:"):
                src = line.split(":", 1)[1].strip()
            if line.startswith("traffic_bytes_per_launch:"):
                traffic = float(line.split(":", 1)[1].strip())
    return traffic if src == sha else None


class ClockSampler:
    """nvidia-smi clock / throttle sampling (every 100 ms) around the timed region.

    Output goes to a file (nvidia-smi buffers its output when piped) and the
    sampler is stopped with SIGINT so the last lines are flushed."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        import tempfile
        self.index = index
        self.proc = None
        self.path = tempfile.mktemp(prefix="svdq_clocks_", suffix=".csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        import signal
        if self.proc is not None:
            self.proc.send_signal(signal.SIGINT)
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            lines = open(self.path).read().splitlines()
            os.unlink(self.path)
        except Exception:
            lines = []
        for line in lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank helpers (one process per GPU; plain replicas, no data collective)
# ---------------------------------------------------------------------------

def max_over_ranks(x: float, device="cpu") -> float:
    """Largest value of `x` over all ranks (device time of the slowest rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: float, steps: int, total_ms: float) -> float:
    """Whole-job TFLOP/s: every rank ran `steps` steps; time = the slowest rank's."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# native (CUDA) arm
# ---------------------------------------------------------------------------

def _run_for(seconds, flush, step):
    """Untimed repetitions of the step (with flushes) for about `seconds`."""
    import torch
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for _ in range(10):
            flush.zero_()
            step()
        torch.cuda.synchronize()

def act_kernel_name(M, K, r, int4, sms=148):
    """The activation kernel the forward runs (the library's routing rule): the
    tensor-core one when r > 0 and each of its 128-row CTAs, K split up to 8
    ways at two CTAs per SM, walks at least 12 stages of 64 columns."""
    if int4:
        return "act_quant_int4_kernel"
    blocks = (M + 127) // 128
    ks = 1
    for c in range(2, 9):
        if K % (64 * c) == 0 and blocks * c <= 2 * sms:
            ks = c
    return "act128_kernel" if r > 0 and K // (64 * ks) >= 12 else "act_quant_kernel"


def kernel_rooflines(M, N, K, r, gemm_ms, act_ms, int4, workload):
    """Roofline entries of the GEMM (the dominant kernel) and the activation
    kernel from their event-timed launch durations (ms): algorithmic bytes or
    flops per launch over the duration, against the measured peaks."""
    flops = 2.0 * M * N * K
    peaks, peak_kind = _peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    # scale bytes per element: one E4M3 per 16 (NVFP4) or one fp16 per 64 (INT4)
    sc_div = 32 if int4 else 16
    act_bytes = M * K * 2 + K * 4 + K * r * 2 + M * K // 2 + M * K // sc_div + M * r * 2
    act_gbs = act_bytes / (act_ms * 1e-3) / 1e9
    # the GEMM's own algorithmic bytes: activation codes, scales and D in; the
    # weight's codes, scales, L2^T and bias in; Y out
    gemm_bytes = (M * K // 2 + M * K // sc_div + M * r * 2 + N * K // 2 + N * K // sc_div + N * r * 2
                  + N * 2 + M * N * 2)
    ridge = fp4_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)        # flop per byte
    if int4:
        i8_peak = peaks["bf16_tflops"] * I8_OVER_BF16
        roofline = {
            "kernel": "int4_gemm_kernel", "bound": "tensor", "achieved": round(gemm_tflops, 1),
            "peak": round(i8_peak, 1), "unit": "TFLOP/s", "frac": round(gemm_tflops / i8_peak, 4),
            "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} x nominal int8:bf16 ratio 2",
            "algorithmic_flops_per_launch": flops,
        }
    elif flops / gemm_bytes >= ridge:
        roofline = {
            "kernel": "fp4_gemm_kernel", "bound": "tensor", "achieved": round(gemm_tflops, 1),
            "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4),
            "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} x nominal fp4:bf16 ratio 4",
            "frac_of_fp4_spec_9pf": round(gemm_tflops / FP4_SPEC_TFLOPS, 4),
            "algorithmic_flops_per_launch": flops,
        }
    else:   # below the ridge (small M): weight streaming, against HBM
        gemm_gbs = gemm_bytes / (gemm_ms * 1e-3) / 1e9
        roofline = {
            "kernel": "fp4_gemm_kernel", "bound": "hbm", "achieved": round(gemm_gbs, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(gemm_gbs / peaks["hbm_gbs"], 4),
            "peak_source": f"{peak_kind} HBM copy",
            "frac_of_hbm_spec_8000": round(gemm_gbs / HBM_SPEC_GBS, 4),
            "tflops": round(gemm_tflops, 2),
        }
    roofline.update({
        "traffic": (_profile_traffic(INT4_SRC, f"int4_gemm_{workload}.txt") if int4 else
                    _profile_traffic(GEMM_SRC, f"fp4_gemm_{workload}.txt")),
        "algorithmic_bytes_per_launch": gemm_bytes,
        "arithmetic_intensity_flop_per_byte": round(flops / gemm_bytes, 1),
        "launch_us": round(gemm_ms * 1e3, 2),
    })
    act_kernel = act_kernel_name(M, K, r, int4)
    if int4:
        act_traffic = _profile_traffic(INT4_SRC, f"act_quant_int4_{workload}.txt")
    elif act_kernel == "act128_kernel":
        act_traffic = _profile_traffic(A128_SRC, f"act128_{workload}.txt")
    else:
        act_traffic = _profile_traffic(ACT_SRC, f"act_quant_{workload}.txt")
    act = {"kernel": act_kernel, "bound": "hbm",
           "achieved": round(act_gbs, 1),
           "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(act_gbs / peaks["hbm_gbs"], 4),
           "algorithmic_bytes_per_launch": act_bytes, "launch_us": round(act_ms * 1e3, 2),
           "traffic": act_traffic}
    return roofline, act, fp4_peak


def few_token_roofline(M, N, K, r, layer_ms, workload, general=None):
    """HBM roofline of one few-token layer call (both of its kernels): the
    algorithmic bytes (X, the weight's codes, scales, L1, L2, 1/lambda and bias,
    and Y, each once) over the per-layer time."""
    peaks, peak_kind = _peaks()
    alg = (M * K * 2 + N * K // 2 + N * K // 16 + K * r * 2 + N * r * 2 + K * 4 + N * 2 + M * N * 2)
    gbs = alg / (layer_ms * 1e-3) / 1e9
    src = [os.path.join(_CSRC, f) for f in ("small_m.cuh", "ptx.cuh", "nvfp4.cuh")]
    out = {"kernel": "act_quant_small_kernel + fp4_gemm_small_m_kernel (one layer call)", "bound": "hbm",
           "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": f"{peak_kind} HBM copy",
           "frac_of_hbm_spec_8000": round(gbs / HBM_SPEC_GBS, 4),
           "traffic": _profile_traffic(src, "small_m_kernels.txt") if workload == "small_m" else None,
           "algorithmic_bytes_per_launch": alg, "launch_us": round(layer_ms * 1e3, 2),
           "tflops": round(2.0 * M * N * K / (layer_ms * 1e-3) / 1e12, 2)}
    if general is not None:
        out["general_path_gemm_alone"] = {k: general.get(k) for k in ("achieved", "unit", "frac", "launch_us")}
    return out


def _time_steps(step, flush, steps, warmup, st):
    """Device time (ms) of each of `steps` calls of step(), L2 flushed before each."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record(st)
        step()
        ev[i][1].record(st)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def _l2_bytes():
    import torch
    try:
        return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)
    except Exception:
        return 126 << 20


class LayerCopies:
    """`n` independent copies of one prepared layer (weight buffer, input,
    output, workspace), so that consecutive steps touch different memory and
    the steps' inputs together exceed L2 (a copy of the weight is a plain
    device copy of the prepared buffer, bound again)."""

    def __init__(self, lin, X, M, n):
        import torch
        import w4a4_rank_corrected_act_b200 as svdq
        self.M, self.N, self.K = M, lin.N, lin.K
        nb = lin.workspace_bytes(M)
        self.nb = nb
        self.items = []
        for i in range(n):
            if i == 0:
                buf, w, Xi = lin.buf, lin.w, X
            else:
                buf = lin.buf.clone()
                w = svdq.svdq_weight_bind_format(buf.data_ptr(), buf.numel(), lin.N, lin.K, lin.r,
                                                 int(lin.has_bias), svdq.FORMAT_NAMES[lin.format])
                Xi = X.clone()
            Yi = torch.empty((M, lin.N), dtype=torch.int16, device="cuda")
            wsi = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
            self.items.append((buf, w, Xi, Yi, wsi))

    @staticmethod
    def count(footprint_bytes, lo=2, hi=16):
        """Copies whose footprints together exceed twice the L2 cache."""
        return int(min(hi, max(lo, -(-2 * _l2_bytes() // max(footprint_bytes, 1)))))

    def step(self, i, sh):
        import w4a4_rank_corrected_act_b200 as svdq
        _, w, X, Y, ws = self.items[i % len(self.items)]
        svdq.svdq_linear_forward(X.data_ptr(), self.M, w, Y.data_ptr(), ws.data_ptr(), self.nb, sh)


def time_back_to_back(step, steps, warmup, st):
    """Device time (ms) of `steps` calls step(i) issued back to back on `st`,
    the sequence captured once in a CUDA graph and replayed (so that host
    launch overhead does not pace the GPU); falls back to eager launches if
    capture fails.  Returns (total_ms, graph_used)."""
    import torch
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    g = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for i in range(steps):
                step(i)
        g.replay()
        torch.cuda.synchronize()
    except Exception:
        g = None
        torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    if g is not None:
        g.replay()
    else:
        for i in range(steps):
            step(i)
    b.record(st)
    torch.cuda.synchronize()
    used = g is not None
    del g
    return a.elapsed_time(b), used


def layer_entry(spec, step_ms):
    """Per-workload entry of the bench line: layer latency percentiles, 4-bit
    TFLOP/s and roofline fractions.  Below the ridge (few tokens) the layer
    is weight streaming and its fraction is taken against HBM with the
    algorithmic bytes (X, the weight's codes, scales, L1, L2, 1/lambda and
    bias, and Y, each once)."""
    peaks, kind = _peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    p50 = float(np.percentile(step_ms, 50))
    tflops = 2.0 * M * N * K / (p50 * 1e-3) / 1e12
    alg_bytes = (M * K * 2 + N * K // 2 + N * K // 16 + K * r * 2 + N * r * 2 + K * 4 + N * 2 + M * N * 2)
    e = {"M": M, "K": K, "N": N, "r": r,
         "us_per_layer": round(p50 * 1e3, 2),
         "us_p95": round(float(np.percentile(step_ms, 95)) * 1e3, 2),
         "tflops": round(tflops, 1),
         "frac_fp4_measured": round(tflops / fp4_peak, 4),
         "frac_fp4_spec_9000": round(tflops / FP4_SPEC_TFLOPS, 4),
         "algorithmic_bytes": alg_bytes}
    ai = 2.0 * M * N * K / alg_bytes
    if ai < fp4_peak * 1e12 / (peaks["hbm_gbs"] * 1e9):
        gbs = alg_bytes / (p50 * 1e-3) / 1e9
        e.update({"bound": "hbm", "gbs": round(gbs, 1), "frac_hbm_measured": round(gbs / peaks["hbm_gbs"], 4),
                  "frac_hbm_spec_8000": round(gbs / HBM_SPEC_GBS, 4),
                  "target_us_70pct_of_8000": round(alg_bytes / (0.7 * HBM_SPEC_GBS * 1e9) * 1e6, 2)})
    else:
        e.update({"bound": "tensor",
                  "target_us_60pct_of_9000": round(2.0 * M * N * K / (0.6 * FP4_SPEC_TFLOPS * 1e12) * 1e6, 2)})
    e["peak_source"] = kind
    return e


def measure_configs(names, steps, warmup, st, flush):
    """Each named workload as one svdq_linear_forward per step on its own
    seeded inputs (weights prepared untimed): `steps` steps back to back over
    rotating copies (inputs beyond L2; the per-layer figure), and the same
    layer alone with L2 flushed before it (the isolated latency)."""
    import torch
    import w4a4_rank_corrected_act_b200 as svdq
    from workloads import gen
    sh = int(st.cuda_stream)
    out = {}
    for name in names:
        spec = gen.workload(name)
        d = gen.make_linear(spec)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa: E731
        lin = svdq.SvdqLinear(dev(d["W"]), torch.from_numpy(d["lam"]).cuda(), dev(d["bias"]), r=spec.r)
        X = dev(d["X"])
        foot = X.numel() * 2 + lin.buf.numel() + lin.workspace_bytes(spec.M) + spec.M * spec.N * 2
        cp = LayerCopies(lin, X, spec.M, LayerCopies.count(foot))
        total_ms, graph = time_back_to_back(lambda i: cp.step(i, sh), steps, warmup, st)
        iso = _time_steps(lambda: cp.step(0, sh), flush, steps, warmup, st)
        e = layer_entry(spec, [total_ms / steps])
        e.update({"copies": len(cp.items), "graph": graph,
                  "us_isolated_p50": round(float(np.percentile(iso, 50)) * 1e3, 2)})
        out[name] = e
        del lin, X, cp
        torch.cuda.empty_cache()
    return out


def measure_mlp_pair(steps, warmup, st, flush):
    """The MLP pair at 1024 x 1024 (up 3072 -> 12288, GELU, down 12288 -> 3072,
    M = 4608, r = 32) through svdq_mlp_forward: back to back over rotating
    copies, and alone with L2 flushed.  The down-projection's smoothing
    factors come from its own input recipe (GELU of a normal draw)."""
    import torch
    import w4a4_rank_corrected_act_b200 as svdq
    from workloads import gen
    sh = int(st.cuda_stream)
    su, sd = gen.workload("mlp_up"), gen.workload("mlp_down")
    du, dd = gen.make_linear(su), gen.make_linear(sd)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa: E731
    up = svdq.SvdqLinear(dev(du["W"]), torch.from_numpy(du["lam"]).cuda(), dev(du["bias"]), r=su.r)
    down = svdq.SvdqLinear(dev(dd["W"]), torch.from_numpy(dd["lam"]).cuda(), dev(dd["bias"]), r=sd.r)
    M, K, F, N = su.M, su.K, su.N, sd.N
    nb = svdq.svdq_mlp_workspace_bytes(M, K, F, N, su.r, sd.r)
    X = dev(du["X"])
    copies = []
    for i in range(2):
        copies.append((X if i == 0 else X.clone(), torch.empty((M, N), dtype=torch.int16, device="cuda"),
                       torch.empty(nb, dtype=torch.uint8, device="cuda")))

    def step(i):
        Xi, Yi, wsi = copies[i % len(copies)]
        svdq.svdq_mlp_forward(Xi.data_ptr(), M, up.w, down.w, Yi.data_ptr(), 0, wsi.data_ptr(), nb, sh)

    total_ms, graph = time_back_to_back(step, steps, warmup, st)
    iso = _time_steps(lambda: step(0), flush, steps, warmup, st)
    flops = 2.0 * M * K * F + 2.0 * M * F * N
    us = total_ms / steps * 1e3
    out = {"M": M, "K": K, "F": F, "N": N, "r": su.r, "us_per_pair": round(us, 2),
           "tflops": round(flops / (us * 1e-6) / 1e12, 1),
           "us_isolated_p50": round(float(np.percentile(iso, 50)) * 1e3, 2), "graph": graph,
           "kernels_per_pair": 4 if sd.r else 3}
    del copies
    # The same pair unfused, for comparison: the two layers through
    # svdq_linear_forward with H = GELU-tanh(Y_up) in bf16 between them (that
    # one elementwise pass is PyTorch's, not this library's: a comparison leg).
    nbu, nbd = up.workspace_bytes(M), down.workspace_bytes(M)
    ucopies = []
    for i in range(2):
        ucopies.append((X if i == 0 else X.clone(), torch.empty((M, F), dtype=torch.bfloat16, device="cuda"),
                        torch.empty((M, N), dtype=torch.int16, device="cuda"),
                        torch.empty(nbu, dtype=torch.uint8, device="cuda"),
                        torch.empty(nbd, dtype=torch.uint8, device="cuda")))

    def ustep(i):
        Xi, Hi, Yi, wu, wd = ucopies[i % len(ucopies)]
        svdq.svdq_linear_forward(Xi.data_ptr(), M, up.w, Hi.data_ptr(), wu.data_ptr(), nbu, sh)
        torch.ops.aten.gelu_(Hi, approximate="tanh")
        svdq.svdq_linear_forward(Hi.data_ptr(), M, down.w, Yi.data_ptr(), wd.data_ptr(), nbd, sh)

    utotal, _ = time_back_to_back(ustep, steps, warmup, st)
    uus = utotal / steps * 1e3
    out["unfused_with_gelu"] = {"us_per_pair": round(uus, 2), "tflops": round(flops / (uus * 1e-6) / 1e12, 1),
                                "note": "svdq_linear_forward (up), PyTorch GELU-tanh in bf16, "
                                        "svdq_linear_forward (down)"}
    del up, down, ucopies
    torch.cuda.empty_cache()
    return out


def run_mlp_pair(args):
    """--mlp-pair: the fused MLP pair alone (svdq_mlp_forward), one JSON line."""
    import torch
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    st = torch.cuda.Stream()
    torch.cuda.set_stream(st)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    pair = measure_mlp_pair(args.steps, args.warmup, st, flush)
    print(json.dumps({"metric": "SVDQ W4A4 MLP pair (up, GELU, down) TFLOP/s", "value": pair["tflops"],
                      "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                      "higher_is_better": True, "dtype": "nvfp4", "data": "synthetic",
                      "config": {"workload": "mlp pair at 1024x1024", "M": pair["M"], "K": pair["K"],
                                 "F": pair["F"], "N": pair["N"], "r": pair["r"]},
                      "mlp_pair_fused": pair}), flush=True)
    return 0


def run_native(args):
    import torch
    import torch.distributed as dist

    import w4a4_rank_corrected_act_b200 as svdq
    from workloads import gen

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    spec = gen.workload(args.workload)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    d = gen.make_linear(spec)
    # a stream of our own (the legacy default stream cannot be captured in a graph)
    st = torch.cuda.Stream()
    torch.cuda.set_stream(st)
    sh = int(st.cuda_stream)

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()

    int4 = args.format == "int4"
    lin = svdq.SvdqLinear(dev(d["W"]), torch.from_numpy(d["lam"]).cuda(), dev(d["bias"]), r=r,
                          format=args.format)
    X = dev(d["X"])
    nb = lin.workspace_bytes(M)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    # consecutive steps use different copies of the weight, input, output and
    # workspace, whose footprints together exceed twice the L2 cache
    foot = X.numel() * 2 + lin.buf.numel() + nb + M * N * 2
    cp = LayerCopies(lin, X, M, LayerCopies.count(foot))
    _, _, _, Y, ws = cp.items[0]

    def step_i(i):
        cp.step(i, sh)

    for i in range(args.warmup):
        step_i(i)
    torch.cuda.synchronize()
    svdq.svdq_clear_device_status(sh)
    # the K timed steps, captured once as one CUDA graph (host launch overhead
    # would otherwise pace the GPU for the shorter layers)
    graph = None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=st):
            for i in range(args.steps):
                step_i(i)
    except Exception:
        graph = None
    torch.cuda.synchronize()

    def timed_steps():
        if graph is not None:
            graph.replay()
        else:
            for i in range(args.steps):
                step_i(i)

    def load_for(seconds):
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < seconds:
            timed_steps()
            torch.cuda.synchronize()

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        # the sampler sees >= 0.5 s of this workload before and after the timed steps
        load_for(0.5)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(st)
        timed_steps()
        t_end.record(st)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        load_for(0.5)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), device="cuda")
    # the same layer alone, L2 flushed before each step (latency of one isolated call)
    step_ms = _time_steps(lambda: step_i(0), flush, args.steps, args.warmup, st)
    status = svdq.svdq_get_device_status(sh)
    if status:
        raise SystemExit(f"device status word {status:#x}: a kernel gave up a wait")

    flops = 2.0 * M * N * K
    value = job_throughput(world, flops, args.steps, total_ms)
    ms_per_step = total_ms / args.steps

    # dominant kernel alone: the FP4 GEMM (svdq_gemm on the act kernel's output),
    # and the activation kernel alone, each timed with events on this stream
    # the forward's own activation kernel (svdq_quantize_act_ws: the 16-row
    # kernel or, with enough K per CTA, the one with D on the tensor cores)
    nba = svdq.svdq_act_workspace_bytes(M, K, r)
    aws = torch.empty(nba, dtype=torch.uint8, device="cuda")

    def a(Xp, Mm, w, cp, sp, dp, s_):
        svdq.svdq_quantize_act_ws(Xp, Mm, w, cp, sp, dp, aws.data_ptr(), nba, s_)
    codes_t = torch.empty(svdq.svdq_act_codes_bytes(M, K), dtype=torch.uint8, device="cuda")
    scales_t = torch.empty(svdq.svdq_act_scales_bytes(M, K), dtype=torch.uint8, device="cuda")
    d_t = torch.empty((M, max(r, 1)), dtype=torch.int16, device="cuda")
    codes_p, scales_p, d_p = codes_t.data_ptr(), scales_t.data_ptr(), d_t.data_ptr()
    reps = max(5, args.steps)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(2 * reps)]
    for i in range(reps):
        flush.zero_()
        ev[i][0].record(st)
        a(X.data_ptr(), M, lin.w, codes_p, scales_p, d_p, sh)
        ev[i][1].record(st)
    for i in range(reps):
        flush.zero_()
        ev[reps + i][0].record(st)
        svdq.svdq_gemm(codes_p, scales_p, d_p, M, lin.w, Y.data_ptr(), sh)
        ev[reps + i][1].record(st)
    torch.cuda.synchronize()
    act_ms = statistics.mean(s.elapsed_time(e) for s, e in ev[:reps])
    gemm_ms = statistics.mean(s.elapsed_time(e) for s, e in ev[reps:])
    roofline, act, fp4_peak = kernel_rooflines(M, N, K, r, gemm_ms, act_ms, int4, args.workload)
    if not int4 and 1 <= M <= 32 and K <= 3840 and N // 128 <= torch.cuda.get_device_properties(0).multi_processor_count:
        # the layer's own call took the few-token path (act_quant_small_kernel, then
        # fp4_gemm_small_m_kernel as its programmatic dependent), whose kernels the
        # entries above (the general path's, called separately) do not time: the
        # roofline is that of one layer call, back to back, against HBM
        roofline = few_token_roofline(M, N, K, r, ms_per_step, args.workload, general=roofline)

    # end to end through the public API with host buffers (pinned), per step:
    # H2D of X, the layer, D2H of Y
    Xh = torch.from_numpy(d["X"].view(np.int16).copy()).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.int16).pin_memory()
    Xd = torch.empty((M, K), dtype=torch.int16, device="cuda")
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(args.warmup):
        svdq.svdq_linear_forward_host(Xh.data_ptr(), M, lin.w, Yh.data_ptr(), Xd.data_ptr(),
                                      Y.data_ptr(), ws.data_ptr(), nb, sh)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        e2e_ev[i][0].record(st)
        svdq.svdq_linear_forward_host(Xh.data_ptr(), M, lin.w, Yh.data_ptr(), Xd.data_ptr(),
                                      Y.data_ptr(), ws.data_ptr(), nb, sh)
        e2e_ev[i][1].record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in e2e_ev), device="cuda")
    e2e = {"value": round(job_throughput(world, flops, args.steps, e2e_ms), 2), "unit": UNIT,
           "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
           "ms_per_step": round(e2e_ms / args.steps, 4)}

    configs = None
    if args.configs and world == 1 and spec.name == "qkv" and not int4:
        # every workload of the benchmark set, one layer each (the qkv entry
        # repeats the headline's own steps), the small-token layer against
        # HBM, and one DiT block of four linears
        configs = {"qkv": layer_entry(spec, [ms_per_step])}
        configs["qkv"].update({"copies": len(cp.items), "graph": graph is not None,
                               "us_isolated_p50": round(float(np.percentile(step_ms, 50)) * 1e3, 2)})
        configs.update(measure_configs(["small", "mlp_up", "mlp_down", "small_m"], args.steps, args.warmup,
                                       st, flush))
        configs["mlp_pair_unfused"] = {
            "us": round(configs["mlp_up"]["us_per_layer"] + configs["mlp_down"]["us_per_layer"], 2),
            "note": "up- and down-projection timed as separate layers (GELU between them not included)"}
        configs["mlp_pair_fused"] = measure_mlp_pair(args.steps, args.warmup, st, flush)
        b_ms, b_layers, b_flops, b_tokens, b_b2b = measure_block("b1", args.steps, args.warmup, st, flush)
        configs["block_b1"] = {"tokens": b_tokens, "us_per_block": round(b_b2b * 1e3, 2),
                               "tflops": round(b_flops / (b_b2b * 1e-3) / 1e12, 1),
                               "us_isolated_p50": round(float(np.percentile(b_ms, 50)) * 1e3, 2),
                               "layers_us_isolated": b_layers}
        if svdq.svdq_get_device_status(sh):
            raise SystemExit("a kernel gave up a wait")

    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4" if int4 else "nvfp4",
            "data": "synthetic (seeded DiT-shaped inputs; no checkpoint)",
            "config": {"workload": f"{spec.name}: DiT joint-attention QKV projection at 1024x1024"
                                   if spec.name == "qkv" else spec.name,
                       "M": M, "K": K, "N": N, "r": r, "bias": True, "format": args.format,
                       "l2": f"steps back to back over {len(cp.items)} copies of weight, input, output and "
                             f"workspace ({len(cp.items) * foot / 2**20:.0f} MiB > 2 x L2), no flush; "
                             "isolated latencies flushed (256 MiB write before each step)",
                       "timing": ("the K steps captured as one CUDA graph, replayed between two events"
                                  if graph is not None else "K eager launches between two events"),
                       "parallelism": f"replicas x{world} (token-parallel, no collective)"},
            "pct_fp4_peak": {"of_spec_9000": round(value / FP4_SPEC_TFLOPS, 4),
                             "of_measured_bf16x4": round(value / fp4_peak, 4),
                             # the timed steps follow 0.5 s of the same load, so they run at the
                             # sustained (power-capped) clock: the sustained bf16 figure x 4
                             "of_measured_sustained_bf16x4": _of_sustained(value)} if not int4 else None,
            "us_per_layer": round(ms_per_step * 1e3, 2),
            "isolated_step_us_percentiles": {"p50": round(float(np.percentile(step_ms, 50)) * 1e3, 2),
                                             "p95": round(float(np.percentile(step_ms, 95)) * 1e3, 2)},
            "roofline": roofline,
            "kernels": {"act_quant": act},
            "e2e": e2e,
            "gpu_launches": 2 * args.steps,
            "clocks": clk.summary(),
        }
        if configs is not None:
            out["configs"] = configs
        if args.cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(spec, d, lin.export(), budget_s=args.cpu_seconds,
                                               fmt=args.format)
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


def measure_block(tag, steps, warmup, st, flush):
    """The four linears of one DiT block (workloads block_<tag>_{qkv,out,up,down})
    back to back on one stream, each on its own synthetic input; one step is
    the four layers, L2 flushed between steps.  Returns per-step ms and the
    mean per-layer us."""
    import torch
    import w4a4_rank_corrected_act_b200 as svdq
    from workloads import gen
    names = [f"block_{tag}_{n}" for n in ("qkv", "out", "up", "down")]
    sh = int(st.cuda_stream)
    layers = []
    for nm in names:
        spec = gen.workload(nm)
        d = gen.make_linear(spec)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa: E731
        lin = svdq.SvdqLinear(dev(d["W"]), torch.from_numpy(d["lam"]).cuda(), dev(d["bias"]), r=spec.r)
        X = dev(d["X"])
        Y = torch.empty((spec.M, spec.N), dtype=torch.int16, device="cuda")
        nb = lin.workspace_bytes(spec.M)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        layers.append((spec, lin, X, Y, ws, nb))

    def step(evs=None):
        for i, (spec, lin, X, Y, ws, nb) in enumerate(layers):
            if evs is not None:
                evs[i].record(st)
            svdq.svdq_linear_forward(X.data_ptr(), spec.M, lin.w, Y.data_ptr(), ws.data_ptr(), nb, sh)
        if evs is not None:
            evs[len(layers)].record(st)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    per = [[torch.cuda.Event(enable_timing=True) for _ in range(len(layers) + 1)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        step(per[i])
    torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[-1]) for e in per]
    layer_us = {spec.name: round(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in per) * 1e3, 2)
                for j, (spec, *_) in enumerate(layers)}
    # the blocks back to back (their footprint exceeds L2 on its own), as one graph
    b2b_ms, graph = time_back_to_back(lambda i: step(), steps, warmup, st)
    flops = sum(2.0 * spec.M * spec.N * spec.K for spec, *_ in layers)
    tokens = layers[0][0].M
    del layers
    torch.cuda.empty_cache()
    return step_ms, layer_us, flops, tokens, b2b_ms / steps


def run_block(args):
    """One DiT block's four linears per step (see measure_block).  One GPU."""
    import torch
    import w4a4_rank_corrected_act_b200 as svdq

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    st = torch.cuda.Stream()
    torch.cuda.set_stream(st)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    with ClockSampler(0) as clk:
        step_ms, layer_us, flops, tokens, b2b_ms = measure_block(args.block, args.steps, args.warmup, st, flush)
    if svdq.svdq_get_device_status(int(st.cuda_stream)):
        raise SystemExit("a kernel gave up a wait")
    total_ms = b2b_ms * args.steps
    out = {
        "metric": METRIC + " (DiT block: four linears)", "value": round(flops * args.steps / (total_ms * 1e-3) / 1e12, 2),
        "unit": UNIT, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic (seeded DiT-shaped inputs; no checkpoint)",
        "config": {"workload": f"DiT block, {tokens} tokens: QKV 3072->9216, out 3072->3072, "
                               "up 3072->12288, down 12288->3072, r=32, bias",
                   "l2": "blocks back to back (a block's footprint exceeds L2), one CUDA graph; "
                         "per-layer times from isolated blocks with L2 flushed before each",
                   "parallelism": "replicas x1 (token-parallel, no collective)"},
        "layers_us_isolated": layer_us,
        "step_us_percentiles": {"p50": round(float(np.percentile(step_ms, 50)) * 1e3, 2),
                                "p95": round(float(np.percentile(step_ms, 95)) * 1e3, 2)},
        "gpu_launches": 8 * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(out), flush=True)
    return out


# ---------------------------------------------------------------------------
# CPU oracle timings
# ---------------------------------------------------------------------------

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


class _Int4OracleView:
    """The INT4 oracle under the NVFP4 oracle's function names used below."""

    def __init__(self, m):
        self.linear_forward = m.linear_forward_int4
        self.quantize_act = m.quantize_act_int4
        self.dequantize = m.dequantize_int4


def cpu_baseline(spec, d, exp, budget_s=15.0, rows=256, fmt="nvfp4"):
    """The oracle's forward (activation quantisation, weight dequantisation,
    float64 GEMM, low-rank branch) on a row sample of the workload, repeated
    for about `budget_s` seconds; the weight is the library's exported one."""
    from oracle import int4_ref
    from oracle import svdq_ref
    if fmt == "int4":
        ref = _Int4OracleView(int4_ref)
    else:
        ref = svdq_ref
    prep = dict(inv_lambda=exp["inv_lambda"], L1=exp["L1"], L2t=exp["L2t"],
                w_codes=exp["w_codes"], w_scales=exp["w_scales"], bias=d["bias"])
    X = d["X"][:rows]
    ref.linear_forward(X[:4], prep)          # warm the BLAS / page in
    n, t0 = 0, time.perf_counter()
    while True:
        ref.linear_forward(X, prep)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s or n >= 50:
            break
    flops = 2.0 * rows * spec.N * spec.K * n
    out = {"value": flops / el / 1e12, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{rows} of {spec.M} token rows x {n} repetitions ({el:.1f} s), full K and N; "
                     "oracle forward incl. per-call weight dequantisation"}
    # the same forward by stage (all cores), and on one BLAS thread (a smaller sample)
    Xs = X[:64]
    t0 = time.perf_counter()
    act = ref.quantize_act(Xs, prep["inv_lambda"], prep["L1"])
    t1 = time.perf_counter()
    ref.dequantize(act["x_codes"], act["x_scales"]) @ ref.dequantize(prep["w_codes"], prep["w_scales"]).T
    t2 = time.perf_counter()
    out["stages_s_64_rows"] = {"quantise_x": round(t1 - t0, 4), "dequantise_and_gemm": round(t2 - t1, 4)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            ref.linear_forward(Xs, prep)
            el1 = time.perf_counter() - t0
        out["value_1_thread"] = 2.0 * 64 * spec.N * spec.K / el1 / 1e12
        out["sample_1_thread"] = "64 token rows, one forward"
    except Exception as e:  # threadpoolctl missing or BLAS not controllable
        out["value_1_thread"] = None
        out["sample_1_thread"] = f"not measured ({type(e).__name__})"
    return out


def run_reference(args):
    """The CPU oracle as the reference arm, end to end on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from oracle import int4_ref
    from oracle import svdq_ref
    from workloads import gen
    spec = gen.workload(args.workload)
    d = gen.make_linear(spec)
    if args.format == "int4":
        ref = _Int4OracleView(int4_ref)
        prep = int4_ref.prepare_weight_int4(d["W"], d["lam"], d["bias"], spec.r)   # offline, untimed
    else:
        ref = svdq_ref
        prep = svdq_ref.prepare_weight(d["W"], d["lam"], d["bias"], spec.r)        # offline, untimed
    rows = args.ref_rows
    X = d["X"][:rows]
    for _ in range(args.warmup):
        ref.linear_forward(X, prep)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        ref.linear_forward(X, prep)
        times.append(time.perf_counter() - t0)
    el = sum(times)
    flops = 2.0 * rows * spec.N * spec.K * args.steps
    value = flops / el / 1e12
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded DiT-shaped inputs; no checkpoint)",
        "config": {"workload": f"{spec.name}: DiT joint-attention QKV projection at 1024x1024"
                               if spec.name == "qkv" else spec.name,
                   "M": spec.M, "K": spec.K, "N": spec.N, "r": spec.r, "format": args.format,
                   "parallelism": "host cores (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"{rows} of {spec.M} token rows per step, full K and N"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="qkv")
    ap.add_argument("--format", choices=["nvfp4", "int4"], default="nvfp4",
                    help="4-bit format of the layer (int4: the variant for pre-Blackwell checkpoints)")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the per-workload entries (small, mlp_up, mlp_down, small_m, DiT block)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--block", choices=["b1", "b4"], default=None,
                    help="time the four linears of a DiT block (QKV, out, up, down) back to back "
                         "on one stream (b1: 4608 tokens, b4: 18432) instead of one workload")
    ap.add_argument("--mlp-pair", action="store_true",
                    help="time only the fused MLP pair (svdq_mlp_forward) at 1024x1024")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1 and int(os.environ.get("RANK", "0")) != 0:
        args.cpu_baseline = False
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        raise SystemExit("for --gpus > 1 launch with torch.distributed.run (one rank per GPU)")
    if args.mlp_pair:
        return run_mlp_pair(args)
    if args.block:
        if args.format != "nvfp4":
            raise SystemExit("--block times the NVFP4 layer")
        return run_block(args)
    return run_native(args)


if __name__ == "__main__":
    main()
