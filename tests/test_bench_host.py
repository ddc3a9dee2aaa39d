"""Host-side logic of bench.py, no GPU: the committed profile's DRAM traffic is reported only while
the kernel source it was captured on is unchanged, and the measured peaks are preferred to the
fallback."""
import hashlib
import json

import bench

SOURCES = ("fused.cu", "engine.cuh", "ptx.cuh", "gemm.cuh")


def _fake_tree(root):
    csrc = root / "quantized_base_lora_nf4_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in SOURCES:
        (csrc / f).write_text(f"// {f}\n")
    dig = hashlib.sha256()
    for f in SOURCES:
        dig.update((csrc / f).read_bytes())
    (root / "profiles").mkdir()
    (root / "profiles" / "k.md").write_text(
        f"# summary\n\ntraffic_bytes_per_launch: 123456\nfused_source_sha256: {dig.hexdigest()}\n")
    return csrc


def test_profile_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("k.md") == 123456.0
    assert bench.profile_traffic("missing.md") is None
    (csrc / "engine.cuh").write_text("// changed\n")
    assert bench.profile_traffic("k.md") is None


def test_measured_peaks_preferred(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks == bench.PEAKS_FALLBACK
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured" and peaks["bf16_tflops"] == 2.0
