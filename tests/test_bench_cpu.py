"""Host-side pieces of bench.py (CPU only): the DRAM-traffic lookup and the weak-scaling value."""

from __future__ import annotations

import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _table(tmp_path, src_text="kernel v1"):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cu").write_text(src_text)
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    rec = {"source": "k.cu", "sha256": sha, "bytes_per_launch": 1000, "blocks": 10, "capture": "k__w.md"}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k@w": rec, "k@w#every": dict(rec, blocks=1)}))


def test_traffic_exact_scaled_and_stale(tmp_path, monkeypatch):
    _table(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("k", "w", 10) == (1000, "profiles/k__w.md")
    b, note = bench.kernel_traffic("k", "w", 30)              # same capture, 3x the blocks
    assert b == 3000 and note.startswith("scaled by blocks")
    b, note = bench.kernel_traffic("k", "other", 5)           # another workload of the same kernel
    assert b == 500 and note.startswith("scaled by blocks")
    assert bench.kernel_traffic("j", "w", 10) == (None, "no capture")
    (tmp_path / "k.cu").write_text("kernel v2")                # source changed since the capture
    assert bench.kernel_traffic("k", "w", 10) == (None, "kernel changed since the capture")


def test_weak_scaling_value():
    assert bench.weak_scaling_value(16_777_216, 1, 7.0) == 16_777_216 / 7e-3 / 1e6
    assert bench.weak_scaling_value(100, 4, 2.0) == 4 * bench.weak_scaling_value(100, 1, 2.0)
