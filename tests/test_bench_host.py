"""Host-side logic of bench.py that needs no GPU: the choice of tensor peak for the
roofline and the traffic lookup's invalidation when a kernel's sources change."""
from __future__ import annotations

import json
import os

import bench


PK = {"hbm_gbs": 6556.2, "bf16_tflops": 1613.7, "bf16_tflops_sustained": 1342.7, "source": "measured"}


def test_tensor_peak_burst_for_short_uncapped_regions():
    assert bench.tensor_peak(PK, 25.0, []) == (1613.7, "burst")


def test_tensor_peak_sustained_for_long_or_power_capped_regions():
    assert bench.tensor_peak(PK, bench.LONG_STEP_MS, []) == (1342.7, "sustained")
    assert bench.tensor_peak(PK, 10.0, ["sw_power_cap"]) == (1342.7, "sustained")


def test_captured_traffic_tracks_the_source_hash(tmp_path, monkeypatch):
    # a capture is reported only for its workload and while its sources hash as recorded
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    import hashlib
    h = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"gemm_gate_up": {"workload": "olmoe", "bytes_per_launch": 123, "sources": ["k.cu"], "sha256": h}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("gemm_gate_up", "olmoe") == 123
    assert bench.captured_traffic("gemm_gate_up", "qwen") is None
    src.write_text("kernel v2")
    assert bench.captured_traffic("gemm_gate_up", "olmoe") is None


def test_committed_traffic_capture_is_well_formed():
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles", "traffic.json")
    d = json.load(open(path))
    for k, v in d.items():
        if k.startswith("_"):
            continue
        assert v["bytes_per_launch"] > 0 and len(v["sha256"]) == 64 and v["sources"]
