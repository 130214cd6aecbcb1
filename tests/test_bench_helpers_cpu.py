"""Host helpers of bench.py (CPU only): the clock record taken during the timed
region, and the rule that a committed ncu traffic figure is reported only
while the kernel's sources match the capture."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler_with(lines):
    s = bench.ClockSampler()
    s.lines = lines
    return s


def test_clock_summary_takes_the_median_and_collects_active_reasons():
    lines = [
        "0, 1900, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1800, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1, 300, 1965, 80.0, 0x0, Active, Not Active, Not Active, Not Active",   # another GPU
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    got = _sampler_with(lines).summary(0)
    assert got["sm_mhz"] == 1800 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["reasons"] == ["sw_power_cap"]
    everyone = _sampler_with(lines).summary(None)
    assert everyone["samples"] == 4 and "hw_slowdown" in everyone["reasons"]


def test_clock_summary_without_samples():
    got = _sampler_with([]).summary(0)
    assert got == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "lse_merge_w1.md").write_text(
        "# x\n\nkernel_source_hash: abc123\ntraffic_bytes_per_launch: 4567\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="attn_fwd": "abc123")
    assert bench.profiled_traffic("w1", kind="lse_merge") == 4567.0
    assert bench.profiled_traffic("w2", kind="lse_merge") is None          # no capture of that workload
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kind="attn_fwd": "def456")
    assert bench.profiled_traffic("w1", kind="lse_merge") is None          # kernel changed since


def test_every_profiled_kernel_names_existing_sources():
    for kind, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "attention_dit_attn_b200", "csrc", f)), (kind, f)
        assert len(bench.kernel_source_hash(kind)) == 16
