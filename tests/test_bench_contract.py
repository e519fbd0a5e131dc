"""The benchmark's JSON line: the clock summary's host logic (CPU), and one short run of
bench.py on a B200 whose line must carry every key of the reporting contract."""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sampler(samples, t_start, t_timed_end, t_end):
    s = object.__new__(bench.ClockSampler)
    s.samples, s.max_sm, s.err = [], 1965, None
    s.t_start, s.t_timed_end, s.t_end = t_start, t_timed_end, t_end
    for t, sm, pw, rs in samples:
        if t_start <= t <= t_end:
            s.samples.append((t, sm, pw, rs))
    return s


def test_clock_summary_prefers_samples_inside_the_timed_region():
    s = _sampler([(1.0, 1900, 400.0, 0x0), (1.5, 1965, 420.0, 0x0), (2.5, 1500, 430.0, 0x4)],
                 t_start=0.9, t_timed_end=2.0, t_end=3.0)
    c = s.summary()
    assert c["samples_timed_region"] == 2 and c["samples"] == 3
    assert c["sm_mhz"] == (1900 + 1965) / 2               # the median of the timed samples
    assert c["sm_mhz_min"] == 1500 and c["reasons"] == ["sw_power_cap"]
    assert c["sm_max_mhz"] == 1965


def test_clock_summary_falls_back_to_the_adjacent_window():
    s = _sampler([(2.2, 1965, 400.0, 0x0), (2.4, 1950, 410.0, 0x0)],
                 t_start=1.0, t_timed_end=2.0, t_end=3.0)
    c = s.summary()
    assert c["samples_timed_region"] == 0 and c["samples"] == 2
    assert c["sm_mhz"] == (1965 + 1950) / 2
    assert "right after the timed region" in c["source"]


def test_clock_summary_reports_throttle_reasons_by_name():
    s = _sampler([(1.1, 1200, 700.0, 0x8 | 0x40)], t_start=1.0, t_timed_end=2.0, t_end=2.0)
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_weak_scaling_value_counts_every_rank():
    assert bench.aggregate_value(10, 4, 2.0) == pytest.approx(4 * 10 / 2e-3)


@pytest.mark.gpu
def test_bench_line_carries_the_contract_keys():
    r = subprocess.run([sys.executable, "bench.py", "--workload", "c64", "--steps", "3", "--warmup", "3",
                        "--no-extra", "--e2e-steps", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["value"] > 0 and line["ms_per_step"] > 0 and line["gpu_launches"] >= 3
    assert "workload" in line["config"] and "l2" in line["config"]
    rf = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf, k
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and 0 < rf["frac"] < 2
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    e2e = line["e2e"]
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in e2e, k
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert e2e["value"] < line["value"]                    # host copies inside the timed steps
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    ck = line["clocks"]
    for k in ("sm_mhz", "sm_max_mhz", "reasons"):
        assert k in ck, k
