"""bench.py end to end on one GPU (short GPT-2-small run): the JSON line
carries every key of the measurement contract, with consistent values."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_json_line_contract():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--config", "gpt2-small", "--steps", "10",
         "--warmup", "3", "--e2e-steps", "5", "--cpu-seconds", "1"],
        capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
              "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 10 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    flops = d["config"]["flops_per_step"]
    assert d["value"] == pytest.approx(flops / (d["ms_per_step"] / 1e3) / 1e12, rel=1e-6)
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-6)
    # the dominant kernel's rate is its algorithmic flops over its in-step time
    assert r["achieved"] == pytest.approx(r["flops_per_launch"] / (r["ms_per_launch"] / 1e3) / 1e12,
                                          rel=1e-6)
    # in-step kernel times add up to the step
    total = sum(k["ms_per_launch"] * k["launches_per_step"] for k in d["kernels"].values())
    assert total == pytest.approx(d["ms_per_step"], rel=1e-3)
    # a 10-step region is far below a second: the burst peak applies
    assert "burst" in r["peak_source"]
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["sample"]
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
    assert "workload" in d["config"]
    # the planned schedule of each product (GPT-2-small: whole tiles, static)
    assert d["config"]["schedules"] == {k: "whole tiles" for k in ("F1", "F2", "B2", "B3", "B4", "B5")}
    # the step's launch structure at this size: five GEMM launches (B3 and B4
    # share one) and one two-pass pair for both bias gradients
    assert d["gpu_launches"] == 7 * d["steps"]
    assert set(d["kernels"]) == {"F1.col_gemm_bias_gelu", "F2.row_gemm_shard_sum",
                                 "B2.dgrad_gelu_grad", "B3+B4.wgrad_dB_dA",
                                 "B5.dgrad_dX_shard_sum", "B1+B2.db_da_colsum"}
