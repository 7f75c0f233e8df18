"""bench.py host logic on CPU: the clock-sample summary that decides whether a
run was throttled, and the ncu traffic record that is used only while the
kernel sources still match the hash recorded with it."""
import json
import os
import shutil
import time

import pytest

import bench
from video_diffusion_transformer_rms_b200 import traffic


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
    # a copy of the tree's kernel sources and one record under a temporary root
    csrc = os.path.join(bench.ROOT, "video_diffusion_transformer_rms_b200", "csrc")
    dst = tmp_path / "video_diffusion_transformer_rms_b200" / "csrc"
    shutil.copytree(csrc, dst)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"rms_adaln": {"workload": "clip5s", "traffic_bytes_per_launch": 2.5e9,
                         "source_sha256": traffic.source_sha("rms_adaln", str(tmp_path))}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_record("rms_adaln", "clip5s") == pytest.approx(2.5e9)
    assert bench.traffic_record("rms_adaln", "clip15s") is None  # another workload
    # any change to a source the kernel is built from voids the record
    with open(dst / "rms_adaln.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_record("rms_adaln", "clip5s") is None
    assert bench.traffic_record("gate_residual", "clip5s") is None  # no record at all


NCU_CSV = """==PROF== Connected to process 1234
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","1","python","h","void sol::qk::qknorm_rope3d_kernel<...>(sol::QkArgs)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Mbyte","668.10"
"0","1","python","h","void sol::qk::qknorm_rope3d_kernel<...>(sol::QkArgs)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","Mbyte","660.00"
"1","1","python","h","void sol::qk::qknorm_rope3d_kernel<...>(sol::QkArgs)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","Gbyte","0.6719"
"1","1","python","h","void sol::qk::qknorm_rope3d_kernel<...>(sol::QkArgs)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","Command line profiler metrics","dram__bytes_write.sum","byte","664000000"
"""


def test_traffic_record_from_an_ncu_csv(tmp_path):
    # per-launch DRAM bytes from ncu's CSV (units converted, launches
    # averaged), scaled from the captured slice to the full workload
    path = tmp_path / "dram.csv"
    path.write_text(NCU_CSV)
    launches = traffic.parse_ncu_csv(str(path))
    assert len(launches) == 2
    assert launches[0][1:] == pytest.approx((668.10e6, 660.0e6))
    assert launches[1][1:] == pytest.approx((671.9e6, 664.0e6))
    rec = traffic.make_record([(launches, 32768)], "qknorm_rope3d_tab", "clip5s", 4 * 32768,
                              "cmd")
    assert rec["traffic_bytes_per_launch"] == pytest.approx(4 * (670.0e6 + 662.0e6))
    assert rec["captures"][0]["rows"] == 32768
    assert rec["source_sha256"] == traffic.source_sha("qknorm_rope3d_tab")
    # two slices: the line through them, so a constant part (writes still in
    # L2 when the launch ends) is not multiplied by the row ratio
    small = [("k", 100.0, 80.0)]            # 100 rows: 100 B read, 80 B written
    large = [("k", 200.0, 180.0)]           # 200 rows: writes = 100 per 100 rows - 20
    rec2 = traffic.make_record([(small, 100), (large, 200)], "rms_adaln", "clip5s", 1000, "c")
    assert rec2["read_bytes_per_launch"] == pytest.approx(1000.0)
    assert rec2["write_bytes_per_launch"] == pytest.approx(980.0)
    with pytest.raises(ValueError):
        traffic.make_record([([], 1)], "rms_adaln", "clip5s", 1, "cmd")
    with pytest.raises(ValueError):
        traffic.make_record([(small, 100), (large, 100)], "rms_adaln", "clip5s", 1, "cmd")
