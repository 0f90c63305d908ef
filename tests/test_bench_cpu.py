"""Host-side pieces of bench.py (no GPU): the recorded ncu traffic is reported only
while the kernel sources hash to the value it was captured with."""

import os
import shutil

import bench


def _copy_tree(tmp_path):
    root = tmp_path / "repo"
    src = os.path.join(bench.ROOT, "persistent_megakernel_02_b200", "csrc")
    shutil.copytree(src, root / "persistent_megakernel_02_b200" / "csrc")
    (root / "profiles").mkdir()
    return root


def _write(root, workload, sha, per_step):
    (root / "profiles" / f"mk_decode_kernel_{workload}_traffic.txt").write_text(
        "# comment line: ignored\n"
        f"workload: {workload}\nkernel_src_sha256_16: {sha}\n"
        f"dram_bytes_read: 1\ndram_bytes_write: 2\ndram_bytes_per_step: {per_step}\n")


def test_traffic_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_src_hash()
    _write(root, "wl_a", sha, 123456789)
    assert bench.recorded_traffic("wl_a") == 123456789.0
    _write(root, "wl_b", "0" * 16, 5)
    assert bench.recorded_traffic("wl_b") is None
    assert bench.recorded_traffic("no_such_workload") is None
    # any change to a kernel source changes the hash
    f = root / "persistent_megakernel_02_b200" / "csrc" / "mk_plan.h"
    f.write_text(f.read_text() + "\n")
    assert bench.kernel_src_hash() != sha
    assert bench.recorded_traffic("wl_a") is None


def test_clock_summary_parses_nvidia_smi_samples():
    """Median SM clock under load, the maximum, and every throttle reason seen active
    (the fields of ClockSampler.FIELDS, in that order)."""
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 850.5, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert bench.ClockSampler(0).summary()["samples"] == 0
