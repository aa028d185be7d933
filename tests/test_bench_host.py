"""Host-side helpers of bench.py on CPU: the clock record that decides
whether a timed run stands, and the profile-summary lookup behind the
roofline's `traffic` field."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# nvidia-smi --format=csv,noheader,nounits rows of ClockSampler.Q:
# index, clocks.sm, clocks.max.sm, power.draw, reasons.active, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
ROWS_POWER_CAP = [
    "0, 1965, 1965, 640.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
    "0, 1890, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    "0, 1875, 1965, 1001.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
]
ROWS_THERMAL = [
    "0, 1500, 1965, 700.0, 0x0000000000000020, Not Active, Not Active, Active, Not Active",
    "0, 1965, 1965, 700.0, 0x0000000000000008, Active, Not Active, Not Active, Not Active",
]


def _summary(tmp_path, rows, with_power=False):
    s = bench.ClockSampler(0, with_power=with_power)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(rows + ["", "0, [N/A], [N/A], [N/A], x, y, z, w, v"]) + "\n")
    s.proc = object()  # as if nvidia-smi had run
    return s.summary()


def test_power_cap_is_reported_with_the_median_clock(tmp_path):
    out = _summary(tmp_path, ROWS_POWER_CAP, with_power=True)
    assert out["sm_mhz"] == 1890.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w"] == 998.7
    assert not os.path.exists(tmp_path / "clocks.csv")  # the record is removed once read


def test_slowdown_reasons_are_all_reported(tmp_path):
    out = _summary(tmp_path, ROWS_THERMAL)
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert "power_w" not in out


def test_no_sampler_says_so():
    s = bench.ClockSampler(0)
    assert s.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_profile_traffic_needs_the_summary_of_the_current_source(tmp_path, monkeypatch):
    """The roofline's traffic comes from a committed ncu summary only while the
    kernel source still has the hash the summary records."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src = tmp_path / "kv_cache_vector_turboquant_b200" / "csrc"
    src.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (src / "k.cu").write_text("kernel v1\n")
    h = bench._source_hash("k.cu")
    (tmp_path / "profiles" / "k.txt").write_text(f"source_sha256_16: {h}\ndram_bytes_per_launch: 12345\n")
    assert bench._profile_traffic("k.cu", "k.txt") == 12345.0
    (src / "k.cu").write_text("kernel v2\n")
    assert bench._profile_traffic("k.cu", "k.txt") is None
    assert bench._profile_traffic("k.cu", "missing.txt") is None
