"""Host helpers of the benchmark: which launches are event-timed, the HBM
peak it divides by, and when the committed DRAM traffic is reported."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_sampled_layer_and_steps():
    assert bench.timed_layer(36) == 18 and bench.timed_layer(1) == 0
    assert bench.timed_step_stride(36) == 1            # one layer of many, every step
    assert bench.timed_step_stride(1) == bench.TIMED_STEP_STRIDE > 1


def test_peak_measured_fallback_and_unreadable(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (6650.0, "fallback")      # no file
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6549.4, "bf16_tflops": 1590}))
    assert bench.peaks() == (6549.4, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.peaks() == (6650.0, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm": 1}))
    assert bench.peaks() == (6650.0, "fallback")


def test_traffic_only_for_its_source_and_workload(tmp_path, monkeypatch):
    csrc = tmp_path / "slow_sparse_kv_sfi_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = b"// kernel source\n"
    (csrc / "attn.cu").write_bytes(src)
    t = {"workload": "w128", "fast_attn_bytes_per_launch": 123.0,
         "attn_cu_sha256": hashlib.sha256(src).hexdigest()}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(t))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("fast_attn_bytes_per_launch", "w128") == 123.0
    assert bench.kernel_traffic("fast_attn_bytes_per_launch", "w32") is None     # another workload
    assert bench.kernel_traffic("dense_attn_bytes_per_launch", "w128") is None   # not captured
    (csrc / "attn.cu").write_bytes(src + b"// changed\n")
    assert bench.kernel_traffic("fast_attn_bytes_per_launch", "w128") is None    # source changed
