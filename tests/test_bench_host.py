"""Host checks of bench.py that need no GPU: the reference arm (the CPU oracle, timed) prints one
JSON line with the contract's keys, for every variant, and the traffic-record helpers agree
with the kernel names the bench reports."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("variant", ["w4a4", "w8a8", "nvfp4", "mxfp4"])
def test_reference_arm_prints_one_contract_line(variant):
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
         "--steps", "2", "--warmup", "1", "--variant", variant],
        capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["config"]["workload"].startswith("tiny")


def test_unknown_group_is_rejected():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "qkv",
         "--group", "64", "--steps", "1", "--warmup", "0"],
        capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode != 0 and "not one of" in (out.stderr + out.stdout)


def test_traffic_key_names_every_reported_kernel():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.traffic_key("void convrot::quant_detail::rht_quant_reg_kernel<256, 7, 256, 2>(...)") \
        == "rht_quant_kernel"
    assert bench.traffic_key("rht_quant_reg_kernel<256, 127, 256, 2>") == "rht_quant_kernel_i8"
    assert bench.traffic_key("rht_quant_reg_kernel<256, 6, 256, 2>") == "rht_quant_kernel_fp4"
    assert bench.traffic_key("void convrot::gemm_detail::w4a4_gemm_kernel<0>(...)") == "w4a4_gemm_kernel"
    assert bench.traffic_key("w8a8_gemm_kernel<0>") == "w8a8_gemm_kernel"
    assert bench.traffic_key("nvfp4_gemm_kernel<0>") == "nvfp4_gemm_kernel"
    assert bench.traffic_key("void convrot::fp4_detail::nvfp4_gemm_kernel<(GemmOut)0>(...)") \
        == "nvfp4_gemm_kernel"
    assert bench.traffic_key("void convrot::mx_detail::mxfp4_gemm_kernel<(GemmOut)0>(...)") \
        == "mxfp4_gemm_kernel"
    # the forms ncu prints
    assert bench.traffic_key("void fp4_detail::nvfp4_gemm_kernel<0>(CUtensorMap_st, ...)") \
        == "nvfp4_gemm_kernel"
    assert bench.traffic_key("void mx_detail::mxfp4_gemm_kernel<0>(CUtensorMap_st, ...)") \
        == "mxfp4_gemm_kernel"
    assert bench.traffic_key("rht_quant_reg_kernel<256, 5, 256, 2>") == "rht_quant_kernel_mx"
