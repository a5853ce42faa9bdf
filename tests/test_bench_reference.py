"""bench.py's reference arm on CPU: the oracle timed on a bounded sample.

The reference arm runs no CUDA code, so its whole command line runs here:
one JSON line on rank 0 with the same metric, unit, direction and `config`
as the library's arm for that workload, a `cpu_baseline` that says how many
oracle threads ran, and zero host<->device bytes; under torchrun the other
ranks exit 0 without work or output.
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "impl", "config", "cpu_baseline", "e2e"}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(cmd, threads):
    env = dict(os.environ, OMP_NUM_THREADS=str(threads))
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return lines


def _check_line(out, workload, world, threads, steps):
    import bench
    assert KEYS <= set(out), KEYS - set(out)
    assert out["impl"] == "reference" and out["metric"] == bench.METRIC and out["unit"] == "TFLOP/s"
    assert out["higher_is_better"] is True and out["scaling"] == "weak" and out["vs_baseline"] is None
    assert out["n_gpus"] == world and out["steps"] == steps and out["warmup"] == 3
    assert out["value"] > 0 and out["ms_per_step"] > 0
    if workload == "moe_dsv3":
        assert out["config"] == bench.moe_arm_config(world)
        assert out["config"]["rows_padded"] % 128 == 0 and out["config"]["rows_padded"] >= 32768
    else:
        assert out["config"] == bench.dense_arm_config(workload, bench.workload_layers(workload), 128, world)
    cpu = out["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] == threads and cpu["value"] == out["value"]
    assert cpu["unit"] == out["unit"] and "rank 0" in cpu["sample"]
    assert out["e2e"] == {"value": out["value"], "unit": out["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}


def test_reference_arm_dense_line():
    lines = _run([sys.executable, "bench.py", "--impl", "reference", "--workload", "esm2_ffn", "--steps", "2",
                  "--warmup", "3", "--ref-seconds", "5"], 4)
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), "esm2_ffn", 1, 4, 2)


def test_reference_arm_default_workload_is_the_largest_config():
    """With no --workload both arms run the largest single-GPU configuration:
    16384 tokens through the square 12288 layer, float scales."""
    import bench
    layers = bench.workload_layers(bench.DEFAULT_WORKLOAD)
    assert [(g.M, g.K, g.N, g.fmt) for _, g, _ in layers] == [(16384, 12288, 12288, 0)]
    lines = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                  "--ref-seconds", "4"], 4)
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), bench.DEFAULT_WORKLOAD, 1, 4, 1)


def test_reference_arm_moe_line():
    lines = _run([sys.executable, "bench.py", "--impl", "reference", "--workload", "moe_dsv3", "--steps", "2",
                  "--warmup", "3", "--ref-seconds", "5"], 4)
    assert len(lines) == 1
    out = json.loads(lines[0])
    _check_line(out, "moe_dsv3", 1, 4, 2)
    assert "routed rows" in out["cpu_baseline"]["sample"]


def test_reference_arm_two_ranks():
    """Launched as the multi-GPU runs are: rank 0 alone times the oracle and
    prints, reporting the world size; rank 1 exits 0 without output."""
    lines = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                  "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl",
                  "reference", "--workload", "esm2_ffn", "--gpus", "2", "--steps", "1", "--warmup", "3",
                  "--ref-seconds", "4"], 2)
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), "esm2_ffn", 2, 2, 1)


def test_reference_arm_refuses_short_warmup():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_cpu_baseline_legs(orc):
    """The `cpu_baseline` object the library's arm adds at N = 1: bounded,
    and `cores` is the oracle's own thread count."""
    import bench
    for cpu in (bench.cpu_baseline("esm2_ffn", budget_s=0.3), bench.cpu_baseline_moe(budget_s=0.3)):
        assert cpu["kind"] == "oracle" and cpu["unit"] == "TFLOP/s" and cpu["value"] > 0
        assert cpu["cores"] == orc.num_threads() and cpu["rows"] >= 2 and cpu["seconds"] < 30
    assert bench.threads_note(4, 8) and not bench.threads_note(8, 8)
