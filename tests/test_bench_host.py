"""Host-side logic of bench.py, no GPU: the committed capture's DRAM traffic is reported only while the
kernel source it was captured on is unchanged and every launch asked for was captured, the measured peaks
are preferred to the fallback, and the CPU baseline times the oracle with fp32 contractions."""
import json
import os

import bench
from synth import workload

SOURCES = bench.FUSED_SOURCES


def _fake_tree(root, keys):
    csrc = root / "quantized_base_lora_nf4_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in SOURCES:
        (csrc / f).write_text(f"// {f}\n")
    (root / "profiles").mkdir()
    return csrc


def test_profile_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    csrc = _fake_tree(tmp_path, None)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles" / "fused_traffic.json").write_text(json.dumps(
        {"fused_source_sha256": bench.fused_source_sha256(), "bytes_per_launch": {"a": 100.0, "b": 300.0}}))
    assert bench.profile_traffic(["a"]) == 100.0
    assert bench.profile_traffic(["a", "b", "b"]) == 700.0 / 3
    assert bench.profile_traffic(["a", "missing"]) is None
    (csrc / "engine.cuh").write_text("// changed\n")
    assert bench.profile_traffic(["a"]) is None


def test_traffic_keys_name_shape_format_and_tokens():
    spec = workload("lqlora").linears[0]
    k = bench.traffic_key("fwd", spec, 2048)
    assert k.startswith("fwd:4096x4096:nf") and k.endswith(":r64:M2048")
    q = workload("qalora").linears[0]
    assert bench.traffic_key("dx", q, 2048) == "dx:4096x4096:int4g32:r16:M2048"


def test_committed_capture_covers_every_fused_launch_of_the_step_workloads():
    """The committed capture has a key for the forward and the input gradient of every linear of the three
    step workloads (the stack, the QA-LoRA layer, the MLP block), so roofline.traffic is reported for each
    while the capture matches the kernel source."""
    with open(os.path.join(bench.ROOT, "profiles", "fused_traffic.json")) as f:
        have = set(json.load(f)["bytes_per_launch"])
    for name, M in (("lqlora", 2048), ("qalora", 2048), ("mlp7b", 4096)):
        for spec in workload(name).linears:
            for kind in ("fwd", "dx"):
                assert bench.traffic_key(kind, spec, M) in have, (name, kind, spec.name)


def test_measured_peaks_preferred(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks == bench.PEAKS_FALLBACK
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured" and peaks["bf16_tflops"] == 2.0


def test_cpu_baseline_times_quantiser_and_fp32_contractions():
    cb = bench.oracle_tokens_per_s(workload("tiny"), 0, budget_s=0.2)
    assert cb["value"] > 0 and cb["cores"] >= 1 and cb["contractions"] == "fp32"
    assert len(cb["quantize_s"]) == 1 and all(v > 0 for v in cb["quantize_s"].values())
