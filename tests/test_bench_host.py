"""bench.py host logic on CPU: the clock-sample summary that decides whether a
run was throttled, and the ncu traffic record that is used only while the
kernel sources still match the hash recorded with it."""
import os
import shutil
import time

import pytest

import bench


def _line(ts, uuid, sm, smax, reasons=("Not Active",) * 4):
    return ", ".join([time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(ts)) + ".123", "0",
                      uuid, str(sm), str(smax), "900.00", *reasons])


def test_clock_summary_median_window_and_reasons():
    t0 = time.time()
    lines = [
        _line(t0 - 30, "GPU-abc", 100, 1965),                     # before the window
        _line(t0, "GPU-abc", 1700, 1965),
        _line(t0 + 1, "GPU-abc", 1750, 1965,
              ("Not Active", "Not Active", "Not Active", "Active")),  # sw_power_cap
        _line(t0 + 2, "GPU-abc", 1800, 1965),
        _line(t0 + 1, "GPU-other", 300, 1965,
              ("Active", "Active", "Active", "Active")),          # another GPU
        "garbage line",
    ]
    r = bench.ClockSampler.summarise(lines, "abc", t0, t0 + 2)
    assert r["samples"] == 3 and r["sm_mhz"] == 1750.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_hardware_slowdown_and_empty_input():
    t0 = time.time()
    lines = [_line(t0, "GPU-abc", 1200, 1965, ("Active", "Not Active", "Active", "Not Active"))]
    r = bench.ClockSampler.summarise(lines, "abc", t0, t0)
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler.summarise([], "abc", t0, t0)["sm_mhz"] is None


def test_traffic_record_only_while_the_sources_match(tmp_path, monkeypatch):
    # a copy of the tree's kernel sources and one summary under a temporary root
    csrc = os.path.join(bench.ROOT, "video_diffusion_transformer_rms_b200", "csrc")
    dst = tmp_path / "video_diffusion_transformer_rms_b200" / "csrc"
    shutil.copytree(csrc, dst)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha("rms_adaln")
    (tmp_path / "profiles" / "rms_adaln_clip5s.md").write_text(
        f"traffic_bytes_per_launch: 2.5e+09\nsource_sha256: {sha}\n")
    assert bench.traffic_record("rms_adaln", "clip5s") == pytest.approx(2.5e9)
    # any change to a source the kernel is built from voids the record
    with open(dst / "rms_adaln.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_record("rms_adaln", "clip5s") is None
    assert bench.traffic_record("gate_residual", "clip5s") is None  # no summary at all
