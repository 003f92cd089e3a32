"""Host-side logic of bench.py (no GPU): the algorithmic byte counts behind the Stage 0-1
roofline, the traffic record's source check, and the calibrated workload."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_stage01_bytes_of_the_128k_workload():
    cfg = bench.workload_config("prefill128k")
    b = bench.stage01_bytes(cfg)
    T, D = 131072, 128
    k = 2 * T * D * 2                      # both KV heads' keys, bf16
    summ = 2 * (T // 64) * D * 4           # fp32 summaries
    q = 32 * T * D * 2                     # every query head, bf16
    mask = 2 * T * 32 * 8                  # 2048 chunks = 32 words per row
    tau = 2 * T * 4
    assert b == dict(stage0=k + summ, stage1=q + summ + mask + tau)
    # about 1.21 GB, the figure the roofline line reports
    assert abs((b["stage0"] + b["stage1"]) / 1e9 - 1.213) < 0.01


def test_calibrated_gamma_is_used_for_128k():
    with open(bench.GAMMA_FILE) as f:
        g = json.load(f)["gamma"]
    assert bench.workload_config("prefill128k").gamma == float(g)
    assert bench.workload_config("gqa32k").gamma == 1.0


def _write_record(path, sha):
    with open(path, "w") as f:
        json.dump({"k_x": {"w": {"sources": ["attend_fa.cu"], "source_sha256_16": sha,
                                 "bytes_per_launch": 1234}}}, f)


def test_traffic_is_reported_only_for_the_captured_source(tmp_path, monkeypatch):
    src = os.path.join(ROOT, "sparse_hierarchical_attention_stage0_b200", "csrc", "attend_fa.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    rec = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    _write_record(rec, sha)
    assert bench.traffic_for("k_x", "w") == 1234
    _write_record(rec, "0" * 16)                        # counters taken on another source
    assert bench.traffic_for("k_x", "w") is None
    assert bench.traffic_for("k_y", "w") is None        # no record at all
