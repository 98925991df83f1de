"""Host-side arithmetic of bench.py (no GPU): algorithmic bytes/flops of a
step, the unique-KV count of shared-prefix batches, and the scaled DRAM
traffic records."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mla_paged_kv_05_b200 import inputs  # noqa: E402


def test_step_work_single_sequence_closed_form():
    w = inputs.make_workload("w", batch=1, heads=64, q_len=4, seqlens=[1000], seed=1)
    d = bench.step_work(w)
    assert d["kv_bytes"] == 1000 * 1152 == d["unique_kv_bytes"]
    assert d["bytes"] == 1000 * 1152 + 4 * 64 * (1152 + 1024 + 4) + 4 * 16 + 4
    # visible tokens: 997 + 998 + 999 + 1000 per head
    assert d["flops"] == 2 * 64 * 1088 * (997 + 998 + 999 + 1000)


def test_unique_kv_counts_shared_prefix_pages_once():
    w = inputs.make_workload("p", batch=3, heads=16, q_len=1, seqlens=[200, 300, 100], seed=2,
                             shared_prefix_tokens=128)
    d = bench.step_work(w)
    # shared: 2 pages (128 tokens); private: 72 + 172 tokens; the third
    # sequence (100 tokens) lies inside the shared pages.
    assert d["kv_bytes"] == 600 * 1152
    assert d["unique_kv_bytes"] == (128 + 72 + 172) * 1152


def test_recorded_traffic_is_scaled_from_a_smaller_capture(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    rec = {"small": {"kernel_sources": h, "dram_bytes_per_launch": 1000},
           "big": {"scaled_from": "small", "scale": 4.0},
           "stale": {"kernel_sources": "0" * 16, "dram_bytes_per_launch": 5}}
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "k1_dram_traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: h)
    assert bench.recorded_traffic("small") == 1000
    assert bench.recorded_traffic("big") == 4000
    assert bench.recorded_traffic("stale") is None
    assert bench.recorded_traffic("absent") is None


def test_oracle_timing_takes_whole_steps_when_they_fit_the_sample():
    w = inputs.tiny()
    us, sample, cores = bench.time_oracle(w, 0.0)
    assert us > 0 and cores >= 1 and "whole step" in sample
    w = inputs.make_workload("long", batch=1, heads=16, q_len=1, seqlens=[300], seed=3)
    us, sample, _ = bench.time_oracle(w, 0.0, sample_tokens=100)
    assert "extrapolated x3.00" in sample
