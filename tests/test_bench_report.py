"""Host logic of bench.py's per-mode report (no GPU): which bf16 peak a fused-kernel launch is
compared with, and the fractions derived from it."""
import math
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from attn_workloads import WORKLOADS  # noqa: E402

PEAKS = {"hbm_gbs": 6548.0, "bf16": 1653.3, "bf16_sustained": 1389.5, "source": "measured"}
CAPPED = {"reasons": ["sw_power_cap"]}


def _report(mode, fused_ms, clocks, prepass_ms=0.5, gemm=None):
    w = WORKLOADS[5]
    r = {"tflops": 1.0, "ms_per_step": fused_ms + prepass_ms,
         "kernel_ms": [fused_ms] if mode == "bf16_exact" else [prepass_ms, fused_ms]}
    return w, bench._mode_report(w, mode, r, PEAKS, clocks, gemm or {})


def test_flop_formula_of_the_largest_workload():
    # 4 * B * Hq * N^2 * d, halved for the causal mask: 140.7 TFLOP for B1 Hq32 N131072 d128
    w = WORKLOADS[5]
    assert w.flops() == 4 * 1 * 32 * 131072 ** 2 * 128 // 2
    assert math.isclose(w.flops() / 1e12, 140.737, rel_tol=1e-4)


@pytest.mark.parametrize("fused_ms, clocks, basis", [
    (115.0, CAPPED, "sustained"),  # a long launch under the power cap: sustained GEMM rate
    (115.0, {"reasons": []}, "burst"),  # long but never capped
    (0.5, CAPPED, "burst"),  # a short launch runs at burst clocks whatever the record says
    (115.0, None, "burst"),  # no clock record
])
def test_peak_basis_follows_the_launch(fused_ms, clocks, basis):
    w, out = _report("int8_qk", fused_ms, clocks)
    assert out["peak_basis"] == basis
    bf16 = PEAKS["bf16_sustained"] if basis == "sustained" else PEAKS["bf16"]
    fused = w.flops() / (fused_ms * 1e-3) / 1e12
    assert math.isclose(out["fused_tflops"], fused)
    assert math.isclose(out["frac_of_int8_peak"], fused / (2 * bf16))
    assert math.isclose(out["frac_of_mixed_peak"], fused / (bf16 * 4 / 3))
    # both bases are always reported, whichever is the headline one
    assert math.isclose(out["frac_of_int8_burst"], fused / (2 * PEAKS["bf16"]))
    assert math.isclose(out["frac_of_int8_sustained"], fused / (2 * PEAKS["bf16_sustained"]))


def test_each_mode_against_its_own_datasheet_peak():
    w, b = _report("bf16_exact", 130.0, CAPPED)
    assert math.isclose(b["frac_of_bf16_datasheet"], b["fused_tflops"] / 2250.0)
    assert "prepass_ms" not in b
    for mode, key in (("int8_qk", "int8"), ("fp8_qk", "fp8")):
        _, r = _report(mode, 115.0, CAPPED)
        assert math.isclose(r[f"frac_of_{key}_datasheet"], r["fused_tflops"] / 4500.0)


def test_prepass_rate_counts_algorithmic_bytes():
    w, out = _report("int8_qk", 115.0, CAPPED, prepass_ms=0.5)
    nq, nk = w.B * w.Hq * w.N * w.d, w.B * w.Hkv * w.N * w.d
    nbytes = 3 * nq + 3 * nk + 4 * w.B * w.Hq * w.N  # read 16-bit once, write 8-bit codes, lse bias
    assert math.isclose(out["prepass_gbs"], nbytes / 0.5e-3 / 1e9)
    assert math.isclose(out["prepass_frac_of_hbm_peak"], out["prepass_gbs"] / PEAKS["hbm_gbs"])


def test_measured_library_gemm_is_an_extra_denominator():
    _, out = _report("int8_qk", 115.0, CAPPED, gemm={"int8_tops": 3051.8})
    assert math.isclose(out["frac_of_measured_int8_gemm"], out["fused_tflops"] / 3051.8)
    _, out = _report("fp8_qk", 115.0, CAPPED, gemm={})
    assert "frac_of_measured_fp8_gemm" not in out


def test_mufu_floor_is_four_d_flops_per_exponential():
    peaks = dict(PEAKS, sms=148, sm_mhz=1965.0)
    for cfg in (4, 5):  # d = 64 and d = 128
        w = WORKLOADS[cfg]
        r = {"tflops": 1.0, "ms_per_step": 10.0, "kernel_ms": [10.0]}
        out = bench._mode_report(w, "bf16_exact", r, peaks, None, {})
        floor = 4 * w.d * 16 * 148 * 1965e6 / 1e12  # 1.19 PFLOP/s at d = 64, 2.38 at d = 128
        assert math.isclose(out["mufu_floor_tflops"], floor)
        assert math.isclose(out["frac_of_mufu_floor"], out["fused_tflops"] / floor)
    # without an SM count or clock the bound is left out rather than guessed
    _, out = _report("int8_qk", 115.0, CAPPED)
    assert "mufu_floor_tflops" not in out


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores, no GPU) prints one JSON line with
    the keys the benchmark contract asks of the reference arm."""
    import json
    import subprocess

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    run = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=root)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [l for l in run.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in r, key
    assert r["impl"] == "reference" and r["value"] > 0 and r["config"]["workload"] == WORKLOADS[5].name
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["e2e"]["h2d_bytes_per_step"] == 0 and r["e2e"]["d2h_bytes_per_step"] == 0
