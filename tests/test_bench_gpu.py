"""bench.py end to end on the GPU: each workload's JSON line carries the contract's keys (needs a B200)."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"}


def _run(*args):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("workload", ["iq1s_4096x4096_weighted", "choice_iq2xs_4096x4096", "iq1s_decode_1m_blocks"])
def test_bench_line(workload):
    line = _run("--workload", workload, "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert KEYS <= set(line)
    assert line["value"] > 0 and line["e2e"]["value"] > 0 and line["gpu_launches"] > 0
    roof = line["roofline"]
    assert roof["bound"] in ("alu", "hbm") and 0 < roof["frac"] < 1.5
    assert line["config"]["workload"] == workload
    if workload == "iq1s_4096x4096_weighted":
        assert line["decode"]["achieved_gbs"] > 0


def test_bench_fp32_peak_probe():
    line = _run("--workload", "fp32_peak")
    rates = line["rates"]
    assert set(rates) == {"ffma", "ffma2", "candidate_mix", "candidate_mix_ffma2"}
    assert all(v > 0 for v in rates.values()) and line["peak"] == max(rates["ffma"], rates["ffma2"])


def test_bench_default_with_cpu_baseline():
    line = _run("--steps", "3", "--warmup", "3")
    assert line["config"]["workload"] == "iq1s_moe_256x1536x4096"
    assert "measured in this run" in line["roofline"]["peak_basis"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
