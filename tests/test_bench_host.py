"""Host-side logic of bench.py that needs no GPU: the DRAM traffic recorded in the ncu
summaries under profiles/ and how it is scaled to a launch."""
import os

import bench


def _write_summary(root, kernel, workload, sha, traffic, units):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    with open(os.path.join(root, "profiles", f"{kernel}_{workload}.md"), "w") as fh:
        fh.write(f"# `{kernel}` on the `{workload}` workload\n\n")
        fh.write(f"- dram_bytes_per_launch: `{traffic}`\n")
        fh.write(f"- units_per_launch: `{units}` (algorithmic bytes of this launch, from the same command)\n")
        fh.write(f"- sources_sha256: `{sha}`\n")


def test_recorded_traffic_scales_by_units(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_sha256", lambda: "abc")
    _write_summary(str(tmp_path), "k_x", "w", "abc", 1000, 500)
    assert bench.recorded_traffic("k_x", "w", 500) == 1000.0
    assert bench.recorded_traffic("k_x", "w", 250) == 500.0      # a launch with half the units


def test_recorded_traffic_stale_or_missing(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_sha256", lambda: "new")
    _write_summary(str(tmp_path), "k_x", "w", "old", 1000, 500)
    assert bench.recorded_traffic("k_x", "w", 500) is None      # sources changed since the capture
    assert bench.recorded_traffic("k_y", "w", 500) is None      # no summary at all
