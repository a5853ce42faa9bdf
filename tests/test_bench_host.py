"""Host logic behind bench.py's JSON line, on CPU: the clock record, the ncu
traffic record, the peak denominators and the algorithmic byte counts."""
import json
import subprocess

import pytest

import bench
import workloads as W

_POPEN = subprocess.Popen  # the real one: the tests below replace bench.subprocess.Popen (the same module)


class _FakeSmi:
    """Stands in for subprocess.Popen: ignores the nvidia-smi command and
    prints the given lines, as `--format=csv,noheader,nounits -lms` would."""

    def __init__(self, lines):
        self.lines = lines

    def __call__(self, cmd, **kw):
        assert cmd[0] == "nvidia-smi" and "--format=csv,noheader,nounits" in cmd
        return _POPEN(["printf", "%s\\n", *self.lines], **kw)


def test_clock_record_median_under_load_and_reasons(monkeypatch):
    lines = ["1965, 1965, 610.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
             "345, 1965, 120.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",  # idle sample
             "1890, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
             "1950, 1965, [N/A], 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",  # no power
             "[N/A], 1965, 500.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",  # no clock
             "garbage"]
    monkeypatch.setattr(bench.subprocess, "Popen", _FakeSmi(lines))
    c = bench.ClockSampler(0)
    c.start()
    c.thread.join(timeout=10)
    out = c.stop()
    assert out["samples"] == 4 and out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == 1950.0  # median of the loaded samples (above half of max): 1890, 1950, 1965
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 998.0


def test_clock_record_thermal_reasons_are_reported(monkeypatch):
    lines = ["1500, 1965, 700, 0x28, Active, Active, Active, Not Active"]
    monkeypatch.setattr(bench.subprocess, "Popen", _FakeSmi(lines))
    c = bench.ClockSampler(0)
    c.start()
    c.thread.join(timeout=10)
    assert c.stop()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_record_without_nvidia_smi(monkeypatch):
    def missing(*a, **k):
        raise OSError("no nvidia-smi")
    monkeypatch.setattr(bench.subprocess, "Popen", missing)
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()
    assert out["samples"] == 0 and out["sm_mhz"] is None and out["reasons"] == ["nvidia-smi unavailable"]


def _raw_csv(path, rows):
    """An `ncu --page raw --csv` export: header, units row, one row per launch."""
    head = ["ID", "Kernel Name", "gpu__time_duration.sum", "dram__bytes_read.sum", "dram__bytes_write.sum"]
    units = ["", "", "us", "Mbyte", "Kbyte"]
    with open(path, "w") as f:
        for r in [head, units] + rows:
            f.write(",".join(f'"{v}"' for v in r) + "\n")


def test_traffic_record_round_trip_and_staleness(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    csv_path = tmp_path / "raw.csv"
    _raw_csv(csv_path, [
        ["0", "void act_quant_kernel<0, 1, 8>(...)", "10.0", "99.0", "99.0"],          # not a GEMM: skipped
        ["1", "void fg8_gemm_kernel<Cfg<256, 0, 3, 4, 0>>(...)", "35.9", "5.093376", "648.704000"],
        ["2", "void fg8_small_m_kernel<1, 16, 1>(...)", "17.6", "1,017.168896", "0.000000"],
    ])
    bench.record_traffic(str(csv_path), "wl")
    assert bench.recorded_traffic("wl", 0) == pytest.approx(5093376 + 648704)
    assert bench.recorded_traffic("wl", 1) == pytest.approx(1017168896)
    assert bench.recorded_traffic("wl", 2) is None and bench.recorded_traffic("other", 0) is None
    # a second workload under the same sources keeps the first
    _raw_csv(csv_path, [["0", "fg8_gemm_kernel", "1", "1.0", "0.0"]])
    bench.record_traffic(str(csv_path), "wl2")
    assert bench.recorded_traffic("wl", 0) == pytest.approx(5093376 + 648704)
    assert bench.recorded_traffic("wl2", 0) == pytest.approx(1e6)
    # counters taken from other kernel sources are not reported ...
    monkeypatch.setattr(bench, "source_hash", lambda: "changed")
    assert bench.recorded_traffic("wl", 0) is None
    # ... and recording under the new sources drops them
    bench.record_traffic(str(csv_path), "wl2")
    rec = json.load(open(tmp_path / "traffic.json"))
    assert rec["source_hash"] == "changed" and list(rec["workloads"]) == ["wl2"]


def test_committed_traffic_is_reported_only_for_its_kernel_sources():
    """profiles/traffic.json holds positive DRAM byte counts; the bench reports
    them only while the kernel sources are the ones they were taken from, and
    null otherwise."""
    rec = json.load(open(bench.TRAFFIC_FILE))
    assert rec["workloads"]
    fresh = rec["source_hash"] == bench.source_hash()
    for wl, v in rec["workloads"].items():
        assert all(b > 0 for b in v["gemm_dram_bytes"])
        got = bench.recorded_traffic(wl, 0)
        assert (got == v["gemm_dram_bytes"][0]) if fresh else (got is None)


def test_peaks_measured_then_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6551.0, "bf16_tflops": 1644.1}))
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6551.0 and p["bf16_tflops_sustained"] == 1644.1


def test_algorithmic_bytes_of_the_esm2_and_dsv3_layers():
    """The per-launch byte counts the roofline divides, as numbers: ESM-2 W1
    (8176 x 480 -> 1920, float scales: Kb 4, Nb 15) and DeepSeek-V3 up
    (8192 x 7168 -> 18432, UE8M0: Kb 56, Nb 144)."""
    esm = W.ESM_W1
    # xq 3,924,480 + xs 130,816 + Wq 921,600 + ws 240 + y 31,395,840 + bias 3,840
    assert bench.gemm_bytes(esm) == 36_376_816
    # x read 7,848,960 + xq 3,924,480 + xs 130,816
    assert bench.quant_bytes(esm) == 11_904_256
    # W read 1,843,200 + Wq 921,600 + ws 240
    assert bench.weight_quant_bytes(esm, 128) == 2_765_040
    up = W.DSV3_UP
    # xq 58,720,256 + xs 458,752 + Wq 132,120,576 + ws 8,064 + y 301,989,888 + bias 36,864
    assert bench.gemm_bytes(up) == 493_334_400
    assert bench.gemm_flops(up) == 2.0 * 8192 * 18432 * 7168
    # 32 x 32 blocks: ceil(18432/32) x ceil(7168/32) = 576 x 224 one-byte scales
    assert bench.weight_quant_bytes(up, 32) == 3 * 18432 * 7168 + 576 * 224
