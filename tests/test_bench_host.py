"""Host-side pieces of bench.py that need no GPU: the committed DRAM-traffic record
is reported only for the kernel sources it was captured on, and the roofline
peaks come from the measured file (with the stated fallback)."""

import json

import bench


def test_traffic_record_is_consistent():
    """A one-pass capture whose per-launch bytes add up; reported only while the
    kernel sources still hash to the recorded digest (else the bench says null)."""
    rec = json.load(open(bench.TRAFFIC_RECORD))
    assert rec["passes"] == 1
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    if rec["kernel_source_sha256"] == bench.kernel_source_digest():
        assert bench.recorded_traffic() == rec["dram_bytes_per_launch"]
    else:
        assert bench.recorded_traffic() is None


def test_traffic_is_withheld_for_other_sources(tmp_path, monkeypatch):
    rec = json.load(open(bench.TRAFFIC_RECORD))
    rec["kernel_source_sha256"] = "0" * 64
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(path))
    assert bench.recorded_traffic() is None
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic() is None


def test_kernel_digest_covers_every_listed_source(tmp_path, monkeypatch):
    files = []
    for i in range(3):
        f = tmp_path / f"s{i}.cu"
        f.write_text(f"source {i}")
        files.append(str(f))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", files)
    d0 = bench.kernel_source_digest()
    (tmp_path / "s2.cu").write_text("source 2 changed")
    assert bench.kernel_source_digest() != d0


def test_peaks_fall_back_when_the_measured_file_is_absent(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, tf, tf_sus, src = bench.load_peaks()
    assert (hbm, tf, src) == (6650.0, 1590.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}))
    hbm, tf, tf_sus, src = bench.load_peaks()
    assert (hbm, tf, src) == (6000.0, 1500.0, "measured")
