"""bench.py's own arm on the GPU: the JSON line it prints keeps its contract.

A short run of a small workload (the ESM-2 FFN step and the few-token Llama
layers) and of the MoE workload, each checked for the keys and the
relations between them: the whole-job value against the median step time,
the dominant kernel's roofline (achieved / peak = frac), the end-to-end leg
with its host-link bound, the clock record, the launch count and the
per-layer table.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks",
        "per_kernel"}


def _bench(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _check(out, workload, steps):
    import bench
    assert KEYS <= set(out), KEYS - set(out)
    assert out["metric"] == bench.METRIC and out["unit"] == "TFLOP/s" and out["higher_is_better"] is True
    assert out["n_gpus"] == 1 and out["steps"] == steps and out["warmup"] == 3 and out["scaling"] == "weak"
    assert out["config"]["workload"] == workload and out["data"] == "synthetic"
    assert out["value"] > 0 and out["ms_per_step"] > 0
    roof = out["roofline"]
    assert roof["bound"] in ("tensor", "hbm") and roof["unit"] in ("TFLOP/s", "GB/s")
    assert roof["achieved"] > 0 and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    assert 0 < roof["frac"] < 1.3
    e2e = out["e2e"]
    assert e2e["unit"] == "TFLOP/s" and 0 < e2e["value"] <= out["value"] * 1.05
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert e2e["host_link_ms_per_step"] > 0 and 0 < e2e["frac_of_host_link"] < 1.2
    assert e2e["ms_per_step"] >= 0.8 * e2e["host_link_ms_per_step"]
    clk = out["clocks"]
    assert "sm_mhz" in clk and "sm_max_mhz" in clk and isinstance(clk["reasons"], list)
    assert out["gpu_launches"] > 0
    assert out["cpu_baseline"] is None  # --no-cpu-baseline
    assert len(out["per_kernel"]) >= 1


def test_esm2_ffn_line():
    out = _bench("--workload", "esm2_ffn", "--steps", "5", "--warmup", "3", "--no-cpu-baseline")
    _check(out, "esm2_ffn", 5)
    import bench
    # the value is the whole step's FLOPs over the median step time
    flops = sum(2.0 * g.M * g.N * g.K for _, g, _ in bench.workload_layers("esm2_ffn"))
    assert abs(out["value"] - flops / (out["ms_per_step"] * 1e-3) / 1e12) <= 1e-6 * out["value"]


def test_few_token_line():
    _check(_bench("--workload", "llama_m16", "--steps", "5", "--warmup", "3", "--no-cpu-baseline"), "llama_m16", 5)


def test_moe_line():
    out = _bench("--workload", "moe_dsv3", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    _check(out, "moe_dsv3", 3)
