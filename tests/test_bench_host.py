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


def test_union_stats_counts_the_chunks_each_unit_walks():
    import torch
    # 8 tokens of one query chunk (diagonal chunk 5), 4 tokens per unit.  Unit 0's tokens route
    # to {0}, {1}, {0}, {0, 2}: union {0, 1, 2} x 4 tokens = 12 executed pairs for 5 active.
    # Unit 1's tokens all route to {3}: 4 executed for 4 active.
    sets = [{0}, {1}, {0}, {0, 2}, {3}, {3}, {3}, {3}]
    words = torch.tensor([[[[sum(1 << c for c in s) | (1 << 5)] for s in sets]]], dtype=torch.int64)
    u = bench.union_stats(words, chunk_size=64, head_dim=128, G=16, tpt=4)
    assert abs(u["factor"] - 16 / 9) < 1e-12
    assert u["executed_flops"] == 4.0 * 128 * 16 * (64 * 16 + 64 * 8)
    # A ragged last unit: 6 tokens at 4 per unit, the second unit holds 2 tokens.
    u2 = bench.union_stats(words[:, :, :6], chunk_size=64, head_dim=128, G=16, tpt=4)
    assert abs(u2["factor"] - (12 + 2) / (5 + 2)) < 1e-12


def test_tokens_per_tile_follow_the_kernels():
    assert bench.tokens_per_tile("k_attend_fa", 16) == 8
    assert bench.tokens_per_tile("k_attend_tc", 8) == 16
    assert bench.tokens_per_tile("k_attend_pair", 16) == 16
    assert bench.tokens_per_tile("k_attend", 4) == 4
    assert bench.tokens_per_tile("k_attend", 32) == 1


def test_support_histogram_bins_and_quantiles():
    """The support-size histogram counts rows per power-of-two bin and reports quantiles."""
    import torch
    cnt = torch.tensor([0, 1, 1, 2, 3, 5, 40, 40, 40, 5000], dtype=torch.int64)
    h = bench.support_histogram(cnt)
    assert h["rows"] == 10 and h["max"] == 5000
    assert h["bins"] == {"0-0": 1, "1-1": 2, "2-3": 2, "4-7": 1, "32-63": 3, "4096-8191": 1}
    assert h["p50"] == 4.0 and abs(h["mean"] - 513.2) < 1e-9


def test_stage1_score_flops_counts_routable_pairs():
    """Stage 1's score FLOPs: 2 D per (row, routable chunk), routable chunks of row t being
    floor(t / Bc) — checked by brute force on a small shape."""
    import bench
    from dash_inputs import PrefillConfig
    cfg = PrefillConfig("t", 2, 8, 2, 1000, 128, 64, 1.5)
    brute = sum(t // 64 for t in range(1000)) * 2 * 128 * 2 * 2
    assert bench.stage1_score_flops(cfg) == brute
    assert abs(bench.FP32_PEAK_TFLOPS - 148 * 128 * 2 * 1.965e-3) < 1e-9
