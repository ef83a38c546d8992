"""bench.py's bookkeeping that needs no GPU: the roofline denominators come from
MEASURED_PEAKS.json when it exists (else the stated fallback), and the DRAM traffic
of the dominant kernel is reported only while the kernel source still matches the
one the ncu counters were taken from."""
import hashlib
import json
import os

import bench


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._peaks() == (6650.0, 1590.0, 1400.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6457.4, "bf16_tflops": 1662.4,
                                                              "bf16_tflops_sustained": 1400.5}))
    assert bench._peaks() == (6457.4, 1662.4, 1400.5, "measured")


def test_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "diffusion_transformer_w4a4_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "k.cu"
    src.write_text("// kernel v1\n")
    rec = {"k": {"bytes_per_launch": 123456, "kernel_source_sha1": hashlib.sha1(src.read_bytes()).hexdigest()}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench._traffic("k", "k.cu") == 123456
    src.write_text("// kernel v2\n")  # changed since the capture
    assert bench._traffic("k", "k.cu") is None
    assert bench._traffic("other", "k.cu") is None


def test_committed_traffic_record_is_well_formed():
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))["gemm_nvfp4"]
    assert rec["bytes_per_launch"] == rec["dram_read_bytes"] + rec["dram_write_bytes"]
    assert len(rec["kernel_source_sha1"]) == 40
