"""Host-side logic of bench.py that decides what a bench line reports: the
peaks it divides by, the clock record it attaches (and that rejects a run
with a slowdown reason), and the recorded DRAM traffic table.  No GPU."""
import json
import os

import bench


class _Proc:  # stands in for the nvidia-smi sampler process
    pass


def _summary(tmp_path, lines):
    p = tmp_path / "clocks.csv"
    p.write_text("".join(line + "\n" for line in lines))
    cs = bench.ClockSampler(0)
    cs.proc = _Proc()
    cs.path = str(p)
    return cs.summary()


def test_clock_summary_uses_loaded_samples_and_collects_reasons(tmp_path):
    idle = "0, 1965, 1965, 150.5, 0x0, Not Active, Not Active, Not Active, Not Active"
    loaded = [
        "0, 1965, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1905, 1965, 998.7, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1935, 1965, 990.1, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = _summary(tmp_path, [idle, *loaded, "garbage line", "0, x, y"])
    # only the samples under load count (power above 200 W), malformed lines are skipped
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1935.0
    assert s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert not os.path.exists(tmp_path / "clocks.csv")  # the record is removed once read


def test_clock_summary_names_every_slowdown_reason(tmp_path):
    line = "0, 1400, 1965, 700.0, 0x0, Active, Active, Active, Not Active"
    s = _summary(tmp_path, [line])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples_or_sampler(tmp_path):
    assert _summary(tmp_path, ["not, a, sample"]) is None
    cs = bench.ClockSampler(0)  # no nvidia-smi process was started
    assert cs.summary() is None


def test_peaks_prefer_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    fb = bench.peaks()
    assert fb["source"] == "fallback" and fb["hbm_gbs"] == 6650.0 and fb["bf16"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6546.6, "bf16_tflops": 1648.7, "bf16_tflops_sustained": 1352.3}))
    m = bench.peaks()
    assert m == dict(hbm_gbs=6546.6, bf16=1648.7, bf16_sustained=1352.3, source="measured")


def test_recorded_traffic_belongs_to_timed_workloads():
    # every recorded DRAM figure names a workload the bench can time, and is
    # at least the dominant kernel's fp32 output it must write
    for name, traffic in bench.TRAFFIC.items():
        assert name in bench.WORKLOADS, name
        assert traffic > 0
    assert bench.TRAFFIC["llama3_8b_up_proj"] >= 8192 * 14336 * 4 * 0.9
    assert bench.TRAFFIC["deepseek_moe16b_bwd"] >= 64 * 1408 * 2048 * 4 * 0.9
