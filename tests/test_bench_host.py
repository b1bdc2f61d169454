"""bench.py's host logic on the CPU: the DRAM traffic of the backward kernel
is taken from the committed ncu summary only for the workload it was captured
on and only while the kernel sources still hash to the value recorded with
it; the roofline fraction uses the measured peak when the driver's file is
there and says so."""
import json

import bench


def _summary(tmp_path, workload, sha, traffic="123456789"):
    p = tmp_path / "summary.txt"
    p.write_text(f"kernel: k\nworkload: {workload}\nsource_sha256: {sha}\n"
                 f"dram_bytes_per_launch: {traffic}\ncommand: x\n")
    return str(p)


def test_traffic_needs_matching_workload_and_sources(tmp_path, monkeypatch):
    sha = bench.kernel_source_hash()
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", _summary(tmp_path, "wl_a", sha))
    assert bench.profiled_traffic("wl_a") == 123456789
    assert bench.profiled_traffic("wl_b") is None
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", _summary(tmp_path, "wl_a", "0" * 64))
    assert bench.profiled_traffic("wl_a") is None
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", _summary(tmp_path, "wl_a", sha, "n/a"))
    assert bench.profiled_traffic("wl_a") is None
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(tmp_path / "missing.txt"))
    assert bench.profiled_traffic("wl_a") is None


def test_source_hash_covers_every_kernel_source(tmp_path, monkeypatch):
    a, b = tmp_path / "a.cuh", tmp_path / "b.cuh"
    a.write_text("one")
    b.write_text("two")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(a), str(b)])
    h0 = bench.kernel_source_hash()
    b.write_text("two, changed")
    assert bench.kernel_source_hash() != h0


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.measured_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}))
    peaks, src = bench.measured_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == 1000.0
