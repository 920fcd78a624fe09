"""Host logic of bench.py on CPU: the staleness rule of the committed ncu
traffic figures, the CPU-baseline leg for both 4-bit formats, and the JSON
contract of the reference arm (the CPU oracle) on the smallest workload."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import int4_ref  # noqa: E402
from oracle import svdq_ref as ref  # noqa: E402
from workloads import gen  # noqa: E402


def test_profile_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cuh"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    sha = bench._src_sha([str(src)])
    (tmp_path / "profiles" / "k_w.txt").write_text(
        f"header\ncommand: x\nsource_sha: {sha}\ntraffic_bytes_per_launch: 12345\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._profile_traffic([str(src)], "k_w.txt") == 12345.0
    assert bench._profile_traffic([str(src)], "missing.txt") is None
    src.write_text("// kernel v2\n")                        # the kernel changed since the capture
    assert bench._profile_traffic([str(src)], "k_w.txt") is None


def test_activation_traffic_comes_from_the_kernel_that_runs(tmp_path, monkeypatch):
    """The activation entry names the kernel the forward routes to and takes its
    traffic from that kernel's own summary: the 128-row one at mlp_down's K,
    the 16-row one at qkv's."""
    (tmp_path / "profiles").mkdir()
    s16, s128 = tmp_path / "a16.cuh", tmp_path / "a128.cuh"
    s16.write_text("// 16-row\n")
    s128.write_text("// 128-row\n")
    (tmp_path / "profiles" / "act_quant_qkv.txt").write_text(
        f"source_sha: {bench._src_sha([str(s16)])}\ntraffic_bytes_per_launch: 111\n")
    (tmp_path / "profiles" / "act128_mlp_down.txt").write_text(
        f"source_sha: {bench._src_sha([str(s128)])}\ntraffic_bytes_per_launch: 222\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "ACT_SRC", [str(s16)])
    monkeypatch.setattr(bench, "A128_SRC", [str(s128)])
    monkeypatch.setattr(bench, "_peaks", lambda: ({"hbm_gbs": 6557.4, "bf16_tflops": 1629.0}, "measured"))
    _, act, _ = bench.kernel_rooflines(4608, 3072, 12288, 32, 0.08, 0.05, False, "mlp_down")
    assert act["kernel"] == "act128_kernel" and act["traffic"] == 222.0
    _, act, _ = bench.kernel_rooflines(4608, 9216, 3072, 32, 0.07, 0.02, False, "qkv")
    assert act["kernel"] == "act_quant_kernel" and act["traffic"] == 111.0


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_cpu_baseline_leg(fmt):
    spec = gen.workload("small")
    d = gen.make_linear(spec)
    if fmt == "int4":
        prep = int4_ref.prepare_weight_int4(d["W"], d["lam"], d["bias"], spec.r)
    else:
        prep = ref.prepare_weight(d["W"], d["lam"], d["bias"], spec.r)
    exp = {k: prep[k] for k in ("w_codes", "w_scales", "L1", "L2t", "inv_lambda")}
    out = bench.cpu_baseline(spec, d, exp, budget_s=0.05, rows=8, fmt=fmt)
    assert out["kind"] == "oracle" and out["unit"] == bench.UNIT
    assert out["value"] > 0 and out["cores"] >= 1
    assert "8 of 256 token rows" in out["sample"]


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_reference_arm_json_line(capsys, fmt):
    out = bench.main(["--impl", "reference", "--workload", "small", "--steps", "1", "--warmup", "3",
                      "--ref-rows", "8", "--format", fmt])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line == json.loads(json.dumps(out))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["config"]["workload"].startswith("small") and line["config"]["format"] == fmt


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--workload", "small", "--warmup", "2"])


def test_kernel_rooflines_for_the_three_regimes():
    peaks, _ = bench._peaks()
    # qkv, NVFP4: above the ridge -> tensor-bound against bf16 burst x 4
    g, a, fp4 = bench.kernel_rooflines(4608, 9216, 3072, 32, 0.0707, 0.0225, False, "qkv")
    assert g["bound"] == "tensor" and g["unit"] == "TFLOP/s" and g["kernel"] == "fp4_gemm_kernel"
    assert fp4 == pytest.approx(peaks["bf16_tflops"] * 4)
    assert g["achieved"] == pytest.approx(2 * 4608 * 9216 * 3072 / 70.7e-6 / 1e12, rel=1e-3)
    assert g["frac"] == pytest.approx(g["achieved"] / g["peak"], rel=1e-3)
    assert g["algorithmic_bytes_per_launch"] == 109725696
    assert a["bound"] == "hbm" and a["algorithmic_bytes_per_launch"] == 36777984
    # small M, NVFP4: below the ridge -> HBM-bound weight streaming
    g, a, _ = bench.kernel_rooflines(16, 18432, 3072, 32, 0.01885, 0.0102, False, "small_m")
    assert g["bound"] == "hbm" and g["unit"] == "GB/s"
    assert g["frac_of_hbm_spec_8000"] == pytest.approx(g["achieved"] / 8000.0, rel=1e-3)
    # INT4 variant: against the 8-bit integer tensor peak (bf16 x 2)
    g, a, _ = bench.kernel_rooflines(4608, 9216, 3072, 32, 0.7394, 0.0353, True, "qkv")
    assert g["kernel"] == "int4_gemm_kernel" and g["peak"] == pytest.approx(peaks["bf16_tflops"] * 2, rel=1e-3)
    assert a["kernel"] == "act_quant_int4_kernel" and a["algorithmic_bytes_per_launch"] == 36335616
    for entry in (g, a):
        t = entry["traffic"]
        assert t is None or t > 0


def test_few_token_roofline_is_one_layer_call_against_hbm():
    peaks, _ = bench._peaks()
    e = bench.few_token_roofline(16, 18432, 3072, 32, 0.0132, "small_m")
    # X, the weight's codes and scales, L1, L2, 1/lambda, bias and Y, each once
    alg = 16 * 3072 * 2 + 18432 * 3072 // 2 + 18432 * 3072 // 16 + 3072 * 32 * 2 + 18432 * 32 * 2 \
        + 3072 * 4 + 18432 * 2 + 16 * 18432 * 2
    assert e["algorithmic_bytes_per_launch"] == alg == 33964032
    assert e["bound"] == "hbm" and e["unit"] == "GB/s" and e["peak"] == peaks["hbm_gbs"]
    assert e["achieved"] == pytest.approx(alg / 13.2e-6 / 1e9, rel=1e-3)
    assert e["frac"] == pytest.approx(e["achieved"] / e["peak"], rel=1e-3)
    t = e["traffic"]
    assert t is None or t > 0


@pytest.mark.parametrize("M,K,r,int4,kernel", [
    (4608, 3072, 32, False, "act_quant_kernel"),      # qkv: a 128-row CTA would walk 6 stages
    (4608, 12288, 32, False, "act128_kernel"),        # mlp_down: 24 stages per CTA at an 8-way split
    (18432, 3072, 32, False, "act128_kernel"),        # 18432 tokens: a 2-way split, 24 stages per CTA
    (256, 512, 32, False, "act_quant_kernel"),        # small: 8 stages in all
    (4608, 12288, 0, False, "act_quant_kernel"),      # no rank-r branch: the 16-row kernel
    (4608, 3072, 32, True, "act_quant_int4_kernel"),
])
def test_activation_kernel_name_follows_the_routing_rule(M, K, r, int4, kernel):
    """The name bench.py reports is the kernel the forward routes to: the
    128-row one when r > 0 and each CTA, with K split up to 8 ways at two CTAs
    per SM, walks at least 12 stages of 64 columns."""
    assert bench.act_kernel_name(M, K, r, int4) == kernel
