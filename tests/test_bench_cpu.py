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


def test_workload_table():
    import ggml_iq_codebook_b200 as iq
    for name, (fmt, shape, text) in bench.WORKLOADS.items():
        assert fmt in iq.IQ_FMT and shape[-1] % 256 == 0 and text, name


def test_reference_arm_prints_the_contract_line():
    """The oracle arm on the host cores (no GPU): one JSON line with the own arm's config."""
    import json
    import subprocess
    env = dict(os.environ, IQ_BENCH_REFERENCE_SECONDS="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3",
                          "--warmup", "3", "--workload", "iq1s_64x256"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads([ln for ln in out.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 3
    assert line["config"]["workload"] == "iq1s_64x256" and line["config"]["format"] == "iq1_s"
    assert line["config"]["shape"] == [64, 256]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
