"""Reporting rules of bench.py that need no GPU: a kernel's DRAM traffic is
reported only while its sources are byte-identical to the ones the capture
was taken with; peaks fall back to the stated figures without the measured
file."""
import hashlib
import json

import bench


def _write_capture(root, sources, nbytes):
    h = hashlib.sha256()
    for rel in sources:
        h.update((root / rel).read_bytes())
    (root / "profiles").mkdir(exist_ok=True)
    entry = {"sources": sources, "bytes_per_launch": nbytes, "sha256": h.hexdigest()}
    (root / "profiles" / "traffic.json").write_text(json.dumps({"kernels": {"k": entry}}))


def test_traffic_reported_until_a_source_changes(tmp_path, monkeypatch):
    (tmp_path / "a.cu").write_text("kernel a\n")
    (tmp_path / "b.cuh").write_text("helpers\n")
    _write_capture(tmp_path, ["a.cu", "b.cuh"], 1234)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("k") == 1234
    assert bench.measured_traffic("other") is None
    with open(tmp_path / "b.cuh", "a") as f:
        f.write("// one more line\n")
    assert bench.measured_traffic("k") is None
    (tmp_path / "b.cuh").unlink()
    assert bench.measured_traffic("k") is None


def test_peaks_fallback_without_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.0,
                                                             "bf16_tflops": 1500.0}))
    p = bench.peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6000.0 and p["bf16_tflops"] == 1500.0
