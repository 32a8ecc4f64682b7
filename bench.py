#!/usr/bin/env python
"""Benchmark of the IQ encoder hot path; rank 0 prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

A step is one pass of the hot path over one batch of synthetic input already resident in HBM.
Default workload: IQ1_S importance-weighted encode of a 4096x4096 bf16 weight (N(0, 0.02^2), 1% of
columns x8, importance = sqrt of a log-normal Hessian diagonal) followed by the decode of its
payload. `value` is weights per second of the whole step (Mweights/s), timed with CUDA events on
the launching stream around the library calls, the L2 cache flushed before every step.

Multi-GPU (torchrun): every rank encodes its own copy of the workload (independent problems, no
data-path collective): weak scaling, time = max over ranks.

--impl reference times the CPU oracle on the host cores (a bounded sample of the same workload per
step); it is the reference arm. It runs on rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ggml_iq_codebook_b200 as iq  # noqa: E402
from ggml_iq_codebook_b200 import synth  # noqa: E402

METRIC = "IQ encode Mweights/s"
UNIT = "Mweights/s"
L2_FLUSH_BYTES = 256 << 20

# FP32 operations the method itself requires (the algorithmic work: every candidate of the
# exhaustive search counts, an fma and a min one op each):
#   IQ1_S, per 8-weight group: 2048 entries x 16 choices = 32,768 candidates x (fma + min) plus
#     about 10 entry-term ops per entry (2048 x 10) = 86,016 ops; per 256-weight block x32 =
#     2,752,512. IQ1_M runs the same search.
#   IQ2_XS, per group: 8,192 candidates x (fma + min) + 512 x 16 fma for A and B = 24,576 ops;
#     per block 786,432. IQ2_S runs it over 1024 entries: 1,572,864 per block.
#   Choice search (G groups of W = 256 / G columns, C choices), per row and block: H Delta
#     (256 x 256 fma) + the own-block scores G x C x (W^2 + W) + two sweeps, each group step
#     counted as C x (W^2 + W) gain products plus a full 256 x W gradient update:
#     65,536 + G C (W^2 + W) + 2 G (C (W^2 + W) + 256 W). IQ2_XS and IQ2_S: 405,504;
#     IQ1_S (8, 32, 16): 602,112; IQ1_M (16, 16, 8): 301,056; eight candidates per 8-weight group
#     (32, 8, 8): 251,904.
OPS_PER_BLOCK = {"iq1_s": 2_752_512, "iq2_xs": 786_432, "iq1_m": 2_752_512, "iq2_s": 1_572_864}


def choice_ops_per_row_block(G: int, C: int = 16) -> int:
    W = 256 // G
    return 256 * 256 + G * C * (W * W + W) + 2 * G * (C * (W * W + W) + 256 * W)


SMS, FP32_LANES = 148, 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}


def alu_peak_tops(mhz: float) -> float:
    return SMS * FP32_LANES * mhz * 1e6 / 1e12


def measure_fp32(dev, kinds=("ffma", "ffma2", "candidate_mix", "candidate_mix_ffma2"), reps=5, iters=200_000):
    """FP32 lane ops/s (T/s) of each probe kind: 8 CTAs of 256 threads per SM, CUDA events on the
    launching stream, median of `reps` launches after one warm-up."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks = 8 * sms
    out = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    rates = {}
    for kind in kinds:
        iq.probe_fp32(kind, blocks, iters // 10, out)
        times = []
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            ops = iq.probe_fp32(kind, blocks, iters, out)
            e.record()
            torch.cuda.synchronize()
            times.append(s.elapsed_time(e))
        rates[kind] = round(ops / (statistics.median(times) / 1e3) / 1e12, 3)
    return rates


def fp32_peak_line(args, dev):
    """--workload fp32_peak: the probe rates as one JSON line, with the clocks seen."""
    with Clocks(torch.cuda.current_device()) as clk:
        rates = measure_fp32(dev)
    clocks = clk.summary()
    nominal = alu_peak_tops(clocks["sm_max_mhz"] if clocks and clocks["sm_max_mhz"] else 1965.0)
    print(json.dumps({"metric": "FP32 lane ops/s", "unit": "Top/s", "rates": rates,
                      "peak": max(rates["ffma"], rates["ffma2"]), "nominal_lanes_x_clock": round(nominal, 3),
                      "clocks": clocks, "probe": "iq_probe_fp32, 8 CTAs x 256 threads per SM, 8 chains/thread"}),
          flush=True)


def kernel_traffic(name: str, workload: str, blocks: int):
    """DRAM bytes (read + write) per launch from a committed ncu capture, if the kernel source is
    unchanged since: the capture of this workload, else one of the same kernel scaled by the blocks
    processed (its traffic grows in proportion). Returns (bytes or None, note)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, "no capture"
    table = json.load(open(path))
    rec = table.get(f"{name}@{workload}")
    scaled = False
    if rec is None:
        cands = [v for k, v in table.items() if k.startswith(name + "@") and "#" not in k]
        if not cands:
            return None, "no capture"
        rec, scaled = cands[0], True
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["sha256"]:
        return None, "kernel changed since the capture"
    if scaled or rec["blocks"] != blocks:
        return int(rec["bytes_per_launch"] * blocks / rec["blocks"]), f"scaled by blocks from profiles/{rec['capture']}"
    return rec["bytes_per_launch"], f"profiles/{rec['capture']}"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, local_index: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [v.strip() for v in vis.split(",")] if vis else None
        self.index = ids[local_index] if ids and local_index < len(ids) else str(local_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.index, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        mhz, maxmhz, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                mhz.append(float(f[1]))
                maxmhz = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": maxmhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest value any rank holds (all_reduce MAX); the value itself on a single process."""
    if dist is None or not dist.is_initialized():
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput in M units/s: every rank processes its own units in the max time."""
    return world * units_per_rank / (ms_per_step_max / 1e3) / 1e6


# ------------------------------------------------------------------------------------ workloads

# workload -> (format, weight shape, description): shared by both arms' JSON config
def _choice_text(fmt: str, shape: str, experts: bool) -> str:
    return (f"local-Hessian choice search, {fmt.upper()}: sqrt(diag H) + one-pass every-choice encode + "
            f"two-sweep search, {shape} bf16 N(0,0.02^2), one H = U^-1 U^-T per "
            + ("expert and " if experts else "") + "256-column block")


WORKLOADS = {
    "iq1s_4096x4096_weighted": ("iq1_s", [4096, 4096], "IQ1_S importance-weighted encode + bf16 decode, 4096x4096 "
                                "bf16 N(0,0.02^2) with 1% columns x8, importance sqrt(lognormal(0,1))"),
    "iq1m_4096x4096_weighted": ("iq1_m", [4096, 4096], "IQ1_M importance-weighted encode + bf16 decode, 4096x4096 "
                                "bf16 N(0,0.02^2) with 1% columns x8, importance sqrt(lognormal(0,1))"),
    "iq2s_8192x4096": ("iq2_s", [8192, 4096], "IQ2_S importance-weighted encode + bf16 decode, 8192x4096 bf16 "
                       "N(0,0.015^2), importance lognormal(0,1)"),
    "iq2xs_8192x4096": ("iq2_xs", [8192, 4096], "IQ2_XS importance-weighted encode + bf16 decode, 8192x4096 bf16 "
                        "N(0,0.015^2), importance lognormal(0,1)"),
    "iq1s_moe_256x1536x4096": ("iq1_s", [256, 1536, 4096], "IQ1_S weighted encode of 256 experts x 1536x4096 bf16 "
                               "in one call + bf16 decode, importance lognormal(0,1) per expert"),
    "iq1s_64x256": ("iq1_s", [64, 256], "IQ1_S encode + bf16 decode, one 64x256 bf16 weight, uniform importance"),
    "choice_iq2xs_4096x4096": ("iq2_xs", [4096, 4096], _choice_text("iq2_xs", "4096x4096", False)),
    "choice_iq2s_4096x4096": ("iq2_s", [4096, 4096], _choice_text("iq2_s", "4096x4096", False)),
    "choice_iq1s_4096x4096": ("iq1_s", [4096, 4096], _choice_text("iq1_s", "4096x4096", False)),
    "choice_iq1m_4096x4096": ("iq1_m", [4096, 4096], _choice_text("iq1_m", "4096x4096", False)),
    "choice_iq2xs_moe_16x1536x4096": ("iq2_xs", [16, 1536, 4096], _choice_text("iq2_xs", "16x1536x4096", True)),
    "choice_iq2xs_g8_4096x4096": ("iq2_xs", [4096, 4096], _choice_text("iq2_xs", "4096x4096", False)
                                  + ", eight candidates (ls 8..15) per 8-weight group over 32 groups of 8 "
                                  "columns, picks only"),
    "choice_iq2xs_4096x4096_per_block": ("iq2_xs", [4096, 4096], _choice_text("iq2_xs", "4096x4096", False)
                                         + ", the search as one call per 256-column block (16 calls)"),
    "iq1s_decode_1m_blocks": ("iq1_s", [4096, 4096], "IQ1_S bf16 decode of 1,048,576 blocks (the 4096x4096 "
                              "weighted payload x16)"),
    "iq2xs_decode_1m_blocks": ("iq2_xs", [8192, 4096], "IQ2_XS bf16 decode of 1,048,576 blocks (the 8192x4096 "
                               "payload x8)"),
    "iq1m_decode_1m_blocks": ("iq1_m", [4096, 4096], "IQ1_M bf16 decode of 1,048,576 blocks (the 4096x4096 "
                              "weighted payload x16)"),
    "iq2s_decode_1m_blocks": ("iq2_s", [8192, 4096], "IQ2_S bf16 decode of 1,048,576 blocks (the 8192x4096 "
                              "payload x8)"),
    "iq1s_decode_4m_blocks": ("iq1_s", [4096, 4096], "IQ1_S bf16 decode of 4,194,304 blocks (the 4096x4096 "
                              "weighted payload x64): a launch whose writes dwarf the L2"),
    "iq2xs_decode_4m_blocks": ("iq2_xs", [8192, 4096], "IQ2_XS bf16 decode of 4,194,304 blocks (the 8192x4096 "
                               "payload x32): a launch whose writes dwarf the L2"),
    "gptq_iq2xs_4096x4096": ("iq2_xs", [4096, 4096], "per-block calibration loop in one call: for each 256-column "
                             "block in order, sqrt(diag H_b) + IQ2_XS every-choice encode + two-sweep local-Hessian "
                             "search + GPTQ propagation of its error to the later columns; 4096x4096 bf16 "
                             "N(0,0.02^2), H^-1 = U^T U whose diagonal blocks give the local-Hessian workload's H_b"),
}


class Workload:
    """Inputs on the device plus one hot-path step; `units` weights per step."""

    def __init__(self, name: str, dev, peaks):
        self.name, self.dev, self.peaks = name, dev, peaks
        self.per_block = False
        self.g8 = "_g8_" in name  # eight candidates per 8-weight group: picks only
        g1 = torch.from_numpy(synth.iq1s_grid()).to(dev)
        g2 = torch.from_numpy(synth.iq2xs_grid()).to(dev)
        g3 = torch.from_numpy(synth.iq2s_grid()).to(dev)
        self.desc = {"iq1_s": iq.make_desc("iq1_s", g1), "iq2_xs": iq.make_desc("iq2_xs", g2),
                     "iq1_m": iq.make_desc("iq1_m", g1), "iq2_s": iq.make_desc("iq2_s", g3)}
        self.launches_per_step = 2
        # the kernels' findings word: kept on the device during the timed steps (no host round
        # trip per call) and checked once afterwards
        self.flags = torch.zeros(1, dtype=torch.int32, device=dev)
        if name not in WORKLOADS:
            raise SystemExit(f"unknown workload {name}")
        text = WORKLOADS[name][2]
        if name == "iq1s_4096x4096_weighted":
            self._encode_decode(synth.workload_iq1s_4096x4096_weighted(), text)
        elif name == "iq1m_4096x4096_weighted":
            self._encode_decode(dict(synth.workload_iq1s_4096x4096_weighted(), fmt="iq1_m"), text)
        elif name == "iq2s_8192x4096":
            self._encode_decode(dict(synth.workload_iq2xs_8192x4096(), fmt="iq2_s"), text)
        elif name == "iq2xs_8192x4096":
            self._encode_decode(synth.workload_iq2xs_8192x4096(), text)
        elif name == "iq1s_moe_256x1536x4096":
            self._encode_decode(synth.workload_iq1s_moe(device=dev), text)
        elif name == "iq1s_64x256":
            self._encode_decode(synth.workload_iq1s_64x256(), text)
        elif name.startswith("choice_"):
            wl = synth.workload_choice_moe() if "moe" in name else synth.workload_choice_iq2xs()
            self._choice(wl, WORKLOADS[name][0], text)
            if name.endswith("_per_block"):
                self.per_block = True
                self.launches_per_step = 2 + self.w.shape[-1] // 256
        elif name.startswith("gptq_"):
            self._gptq(synth.workload_gptq_iq2xs(), text)
        elif name.endswith("m_blocks") and "_decode_" in name:
            base = {"iq1s": synth.workload_iq1s_4096x4096_weighted(), "iq1m": dict(
                synth.workload_iq1s_4096x4096_weighted(), fmt="iq1_m"), "iq2xs": synth.workload_iq2xs_8192x4096(),
                "iq2s": dict(synth.workload_iq2xs_8192x4096(), fmt="iq2_s")}
            self._encode_decode(base[name.split("_")[0]], text)
            self.kind = "decode"
            B = iq.BLOCK_BYTES[self.fmt]
            mblocks = int(name.split("_")[-2][:-1])  # 1 or 4 (x 2^20 blocks)
            self.payload = self.payload.reshape(-1, B).repeat((mblocks << 20) // (self.payload.numel() // B), 1)
            self.decoded = torch.empty((self.payload.shape[0], 256), dtype=torch.bfloat16, device=self.dev)
            self.units = self.payload.shape[0] * 256
            self.nblocks = self.payload.shape[0]
            self.launches_per_step = 1
            self.dominant = "decode_kernel"
            self.ops_per_launch = None

    def _encode_decode(self, wl, text):
        self.fmt = wl["fmt"]
        self.kind = "encode"
        self.w_host = wl["w"]
        self.imp_host = wl["importance"]
        self.w = wl["w"].to(self.dev)
        self.imp = None if wl["importance"] is None else wl["importance"].to(self.dev)
        shape = tuple(self.w.shape[:-1]) + (self.w.shape[-1] // 256, iq.BLOCK_BYTES[self.fmt])
        self.payload = torch.empty(shape, dtype=torch.uint8, device=self.dev)
        self.decoded = torch.empty(tuple(self.w.shape[:-1]) + (self.w.shape[-1],), dtype=torch.bfloat16,
                                   device=self.dev)
        self.units = self.w.numel()
        self.nblocks = self.units // 256
        self.text = text
        self.dominant = "iq2_encode_kernel" if self.fmt in ("iq2_xs", "iq2_s") else "iq1_encode_kernel"
        self.ops_per_launch = self.nblocks * OPS_PER_BLOCK[self.fmt]
        # validate once (findings word + raise) before anything is timed
        iq.iq_encode(self.desc[self.fmt], self.w, self.imp, out=self.payload)

    def _choice(self, wl, fmt, text):
        self.fmt, self.kind = fmt, "choice"
        self.w_host, self.hess_host = wl["w"], wl["hess"]
        self.w, self.hess = wl["w"].to(self.dev), wl["hess"].to(self.dev)
        lead, cols = tuple(self.w.shape[:-1]), self.w.shape[-1]
        nblk = cols // 256
        nexp = lead[0] if len(lead) == 2 else 1
        self.imp = torch.empty((nexp, cols) if len(lead) == 2 else (cols,), dtype=torch.float32, device=self.dev)
        B, G = iq.BLOCK_BYTES[fmt], (32 if self.g8 else iq.CHOICE_GROUPS[fmt])
        self.cand = torch.empty((iq.CHOICES[fmt],) + lead + (nblk, B), dtype=torch.uint8, device=self.dev)
        self.picks = torch.empty(lead + (nblk, G), dtype=torch.uint8, device=self.dev)
        self.picks_b = torch.empty((nblk,) + lead + (1, G), dtype=torch.uint8, device=self.dev)
        self.payload = torch.empty(lead + (nblk, B), dtype=torch.uint8, device=self.dev)
        self.units = self.w.numel()
        self.nblocks = self.units // 256
        self.launches_per_step = 3
        self.text = text
        self.dominant = "choice_search_kernel"
        self.ops_per_launch = self.nblocks * choice_ops_per_row_block(G, 8 if self.g8 else iq.CHOICES[fmt])
        iq.iq_sqrt_diag(self.hess, out=self.imp)
        iq.iq_encode(self.desc[fmt], self.w, self.imp, every_choice=True, out=self.cand)

    def _gptq(self, wl, text):
        self.fmt, self.kind = wl["fmt"], "gptq"
        self.w_host, self.hess_host, self.u_host = wl["w"], wl["hess"], wl["U"]
        self.w, self.hess, self.U = wl["w"].to(self.dev), wl["hess"].to(self.dev), wl["U"].to(self.dev)
        rows, cols = self.w.shape
        nblk = cols // 256
        self.workspace = torch.empty(iq.iq_gptq_workspace_bytes(self.fmt, rows), dtype=torch.uint8, device=self.dev)
        self.payload = torch.empty((rows, nblk, iq.BLOCK_BYTES[self.fmt]), dtype=torch.uint8, device=self.dev)
        self.picks = torch.empty((rows, nblk, iq.CHOICE_GROUPS[self.fmt]), dtype=torch.uint8, device=self.dev)
        self.w_work = torch.empty((rows, cols), dtype=torch.float32, device=self.dev)
        self.units = self.w.numel()
        self.nblocks = self.units // 256
        self.text = text
        self.launches_per_step = 1 + 5 * nblk - 2  # fp32 copy; per block sqrt diag, encode, search, solve, update
        self.dominant = "per-block loop (every kernel of the call)"
        # the algorithmic counts for the encode and the search, plus the propagation: the solve's
        # 256 x 255 / 2 fmas per row-block and rows x 256 fmas per later column
        later = sum(cols - 256 * (b + 1) for b in range(nblk))
        self.ops_per_launch = (self.nblocks * (OPS_PER_BLOCK[self.fmt] + choice_ops_per_row_block(16) + 256 * 255 // 2)
                               + rows * 256 * later)
        self.step()

    # one step; `ev` is a list of (start, end) event pairs to fill around the dominant kernel
    def step(self, ev=None):
        d = self.desc[self.fmt]
        if self.kind == "decode":
            if ev is not None:
                ev[0].record()
            iq.iq_decode(d, self.payload, torch.bfloat16, out=self.decoded)
            if ev is not None:
                ev[1].record()
        elif self.kind == "gptq":
            if ev is not None:
                ev[0].record()
            iq.iq_gptq_blocks(d, self.w, self.hess, self.U, workspace=self.workspace, payload=self.payload,
                              picks=self.picks, w_work=self.w_work, flags=self.flags)
            if ev is not None:
                ev[1].record()
        elif self.kind == "encode":
            if ev is not None:
                ev[0].record()
            iq.iq_encode(d, self.w, self.imp, out=self.payload, flags=self.flags, raise_on_flags=False)
            if ev is not None:
                ev[1].record()
            iq.iq_decode(d, self.payload, torch.bfloat16, out=self.decoded)
        else:
            iq.iq_sqrt_diag(self.hess, out=self.imp)
            iq.iq_encode(d, self.w, self.imp, every_choice=True, out=self.cand, flags=self.flags,
                         raise_on_flags=False)
            if ev is not None:
                ev[0].record()
            if self.per_block:  # one call per 256-column block, on views into the whole-weight tensors
                for b in range(self.w.shape[-1] // 256):
                    iq.iq_choice_search(d, self.w[:, 256 * b:256 * (b + 1)], self.hess[b:b + 1],
                                        self.cand[:, :, b:b + 1], picks=self.picks_b[b],
                                        payload=self.payload[:, b:b + 1], flags=self.flags)
            elif self.g8:
                iq.iq_choice_search_g8(d, self.w, self.hess, self.cand, picks=self.picks, flags=self.flags)
            else:
                iq.iq_choice_search(d, self.w, self.hess, self.cand, picks=self.picks, payload=self.payload,
                                    flags=self.flags)
            if ev is not None:
                ev[1].record()

    def e2e_step(self, host):
        """Same step through the public API from pinned host memory, results read back."""
        d = self.desc[self.fmt]
        if self.kind == "decode":
            self.payload.copy_(host["payload"], non_blocking=True)
            iq.iq_decode(d, self.payload, torch.bfloat16, out=self.decoded)
            host["decoded"].copy_(self.decoded, non_blocking=True)
        elif self.kind == "gptq":
            self.w.copy_(host["w"], non_blocking=True)
            self.hess.copy_(host["hess"], non_blocking=True)
            self.U.copy_(host["U"], non_blocking=True)
            self.step()
            host["payload"].copy_(self.payload, non_blocking=True)
            host["picks"].copy_(self.picks, non_blocking=True)
        elif self.kind == "encode":
            self._e2e_encode_pipelined(d, host)
        else:
            self.w.copy_(host["w"], non_blocking=True)
            self.hess.copy_(host["hess"], non_blocking=True)
            self.step()
            picks = self.picks_b if self.per_block else self.picks
            host["picks"].view(-1).copy_(picks.view(-1), non_blocking=True)
            if not self.g8:
                host["payload"].copy_(self.payload, non_blocking=True)

    def _e2e_encode_pipelined(self, d, host, chunks=16):
        """The encode + decode step from pinned host memory, cut along the leading dimension
        (experts, or rows) into `chunks` pieces that flow through three streams: the host-to-device
        copy of piece i + 1 and the device-to-host copy of piece i - 1 overlap the kernels of
        piece i. Every byte of the step still crosses the bus inside the timed region."""
        if not hasattr(self, "_e2e_streams"):
            self._e2e_streams = (torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev))
        s_in, s_out = self._e2e_streams
        comp = torch.cuda.current_stream(self.dev)
        n = self.w.shape[0]
        step = (n + chunks - 1) // chunks
        per_expert_imp = self.imp is not None and self.imp.dim() == 2
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        if self.imp is not None and not per_expert_imp:
            with torch.cuda.stream(s_in):
                self.imp.copy_(host["imp"], non_blocking=True)
        for i0 in range(0, n, step):
            sl = slice(i0, min(n, i0 + step))
            with torch.cuda.stream(s_in):
                self.w[sl].copy_(host["w"][sl], non_blocking=True)
                if per_expert_imp:
                    self.imp[sl].copy_(host["imp"][sl], non_blocking=True)
            comp.wait_stream(s_in)
            imp = None if self.imp is None else (self.imp[sl] if per_expert_imp else self.imp)
            iq.iq_encode(d, self.w[sl], imp, out=self.payload[sl], flags=self.flags, raise_on_flags=False)
            iq.iq_decode(d, self.payload[sl], torch.bfloat16, out=self.decoded[sl])
            s_out.wait_stream(comp)
            with torch.cuda.stream(s_out):
                host["payload"][sl].copy_(self.payload[sl], non_blocking=True)
                host["decoded"][sl].copy_(self.decoded[sl], non_blocking=True)
        comp.wait_stream(s_out)

    def host_buffers(self):
        pin = lambda t: t.to("cpu").pin_memory()  # noqa: E731
        if self.kind == "decode":
            h = {"payload": pin(self.payload), "decoded": pin(self.decoded)}
            h2d, d2h = self.payload.numel(), self.decoded.numel() * 2
        elif self.kind == "gptq":
            h = {"w": pin(self.w_host), "hess": pin(self.hess_host), "U": pin(self.u_host), "payload": pin(self.payload),
                 "picks": pin(self.picks)}
            h2d = self.w.numel() * 2 + self.hess.numel() * 4 + self.U.numel() * 4
            d2h = self.payload.numel() + self.picks.numel()
        elif self.kind == "encode":
            h = {"w": pin(self.w_host), "payload": pin(self.payload), "decoded": pin(self.decoded)}
            if self.imp is not None:
                h["imp"] = pin(self.imp_host)
            h2d = self.w.numel() * 2 + (0 if self.imp is None else self.imp.numel() * 4)
            d2h = self.payload.numel() + self.decoded.numel() * 2
        else:
            h = {"w": pin(self.w_host), "hess": pin(self.hess_host), "picks": pin(self.picks),
                 "payload": pin(self.payload)}
            h2d = self.w.numel() * 2 + self.hess.numel() * 4
            d2h = self.picks.numel() + (0 if self.g8 else self.payload.numel())
        return h, h2d, d2h


def decode_roofline(wl: Workload, dev, peaks):
    """The decoder timed alone on an HBM-sized input: the workload's payload tiled to ~3.5 GB."""
    if wl.kind not in ("encode", "decode"):
        return None
    B = iq.BLOCK_BYTES[wl.fmt]
    flat = wl.payload.reshape(-1, B)
    reps = max(1, (6 << 20) // flat.shape[0])
    big = flat.repeat(reps, 1)
    out = torch.empty((big.shape[0], 256), dtype=torch.bfloat16, device=dev)
    d = wl.desc[wl.fmt]
    for _ in range(3):
        iq.iq_decode(d, big, torch.bfloat16, out=out)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    times = []
    for _ in range(10):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        iq.iq_decode(d, big, torch.bfloat16, out=out)
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    ms = statistics.median(times)
    nblocks = int(big.shape[0])
    nbytes = nblocks * (B + 512)
    gbs = nbytes / ms / 1e6
    del big, out, flush
    # the DRAM counters of a 4M-block launch where there is one (writes still in the L2 when a
    # launch ends escape its counters, a smaller share of a larger launch), else of a 1M-block one
    name = {"iq1_s": ["iq1s_decode_4m_blocks", "iq1s_decode_1m_blocks"],
            "iq2_xs": ["iq2xs_decode_4m_blocks", "iq2xs_decode_1m_blocks"], "iq1_m": ["iq1m_decode_1m_blocks"],
            "iq2_s": ["iq2s_decode_1m_blocks"]}
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    captured = set(json.load(open(tpath))) if os.path.exists(tpath) else set()
    traffic, note = None, f"no capture of the {wl.fmt} decode"
    for cand in name.get(wl.fmt, []):
        if f"decode_kernel@{cand}" in captured:
            traffic, note = kernel_traffic("decode_kernel", cand, nblocks)
            break
    return {"kernel": "decode_kernel (bf16 out)", "blocks": nblocks, "bytes_per_launch": nbytes,
            "ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "peak_gbs": peaks["hbm_gbs"],
            "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic, "traffic_source": note}


# ------------------------------------------------------------------------------------ oracle arm

def oracle_sample_rate(name: str, budget_s: float, rows_hint: int | None = None):
    """Oracle encode + decode on the first rows of the workload, sized to ~budget_s of wall time."""
    import oracle
    if name.startswith("gptq_"):
        wl = synth.workload_gptq_iq2xs()
        g = synth.iq2xs_grid()
        w, hess, U = wl["w"], wl["hess"].numpy(), wl["U"].numpy()

        def run(r):
            oracle.gptq_blocks("iq2_xs", g, iq.DEFAULT_ANCHOR["iq2_xs"], w[:r], hess, U)
        cols = w.shape[1]
    elif name.startswith("choice_"):
        cfmt = {"choice_iq2xs_4096x4096": "iq2_xs", "choice_iq2s_4096x4096": "iq2_s",
                "choice_iq1s_4096x4096": "iq1_s", "choice_iq1m_4096x4096": "iq1_m",
                "choice_iq2xs_moe_16x1536x4096": "iq2_xs", "choice_iq2xs_4096x4096_per_block": "iq2_xs",
                "choice_iq2xs_g8_4096x4096": "iq2_xs"}[name]
        if "moe" in name:  # the sample is the first rows of expert 0, under its own Hessians
            wl = synth.workload_choice_moe()
            w, hess = wl["w"][0], wl["hess"][0].numpy()
        else:
            wl = synth.workload_choice_iq2xs()
            w, hess = wl["w"], wl["hess"].numpy()
        g = {"iq2_xs": synth.iq2xs_grid, "iq2_s": synth.iq2s_grid, "iq1_s": synth.iq1s_grid,
             "iq1_m": synth.iq1s_grid}[cfmt]()
        imp = oracle.sqrt_diag(hess)

        def run(r):
            cand, _ = oracle.encode(cfmt, g, iq.DEFAULT_ANCHOR[cfmt], w[:r], importance=imp, every_choice=True)
            if "_g8_" in name:
                oracle.choice_search_g8(g, w[:r], hess, cand)
            else:
                oracle.choice_search(cfmt, g, w[:r], hess, cand)
        cols = w.shape[1]
    else:
        if name == "iq1s_moe_256x1536x4096":
            w, imp = synth.expert_bf16(0, 1536, 4096, 0.02, 1004), synth.lognormal((256, 4096), 3004)[0]
            fmt = "iq1_s"
        else:
            wl = {"iq1s_4096x4096_weighted": synth.workload_iq1s_4096x4096_weighted,
                  "iq1m_4096x4096_weighted": synth.workload_iq1s_4096x4096_weighted,
                  "iq1s_decode_1m_blocks": synth.workload_iq1s_4096x4096_weighted,
                  "iq1m_decode_1m_blocks": synth.workload_iq1s_4096x4096_weighted,
                  "iq2xs_decode_1m_blocks": synth.workload_iq2xs_8192x4096,
                  "iq1s_decode_4m_blocks": synth.workload_iq1s_4096x4096_weighted,
                  "iq2xs_decode_4m_blocks": synth.workload_iq2xs_8192x4096,
                  "iq2s_decode_1m_blocks": synth.workload_iq2xs_8192x4096,
                  "iq2xs_8192x4096": synth.workload_iq2xs_8192x4096,
                  "iq2s_8192x4096": synth.workload_iq2xs_8192x4096,
                  "iq1s_64x256": synth.workload_iq1s_64x256}[name]()
            fmt = "iq1_m" if name.startswith("iq1m") else "iq2_s" if name.startswith("iq2s") else wl["fmt"]
            w, imp = wl["w"], wl["importance"]
        g = {"iq2_xs": synth.iq2xs_grid, "iq2_s": synth.iq2s_grid}.get(fmt, synth.iq1s_grid)()

        def run(r):
            p, _ = oracle.encode(fmt, g, iq.DEFAULT_ANCHOR[fmt], w[:r], importance=imp)
            oracle.decode(fmt, g, p)
        cols = w.shape[1]
    total_rows = w.shape[0]
    if rows_hint is None:
        t0 = time.perf_counter()
        run(1)
        t1 = time.perf_counter() - t0
        rows = int(max(1, min(total_rows, budget_s / max(t1, 1e-6))))
    else:
        rows = rows_hint
    t0 = time.perf_counter()
    run(rows)
    dt = time.perf_counter() - t0
    return rows * cols / dt / 1e6, rows, cols, dt, oracle.threads(), run


def reference_arm(args, n_gpus, config):
    import oracle
    rate, rows, cols, dt, cores, run = oracle_sample_rate(args.workload, budget_s=1.0)
    # per step: a bounded sample sized so that warm-up + timed steps take about 90 s in all
    budget = float(os.environ.get("IQ_BENCH_REFERENCE_SECONDS", "90"))
    per_row = dt / rows
    rows = int(max(1, min(rows * 50, budget / (args.steps + args.warmup) / per_row)))
    for _ in range(args.warmup):
        run(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(rows)
    dt = time.perf_counter() - t0
    value = args.steps * rows * cols / dt / 1e6
    sample = f"first {rows} rows x {cols} cols of the workload per step (encode + decode on the host cores)"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": n_gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=80)  # about 53 s of timed work on the default workload
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="own", choices=["own", "reference"])
    ap.add_argument("--workload", default="iq1s_moe_256x1536x4096")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    peaks = load_peaks()
    if args.workload == "fp32_peak":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        iq.load_library()
        if rank == 0:
            fp32_peak_line(args, dev)
        return
    if args.workload not in WORKLOADS:
        raise SystemExit(f"unknown workload {args.workload}")
    fmt, shape, text = WORKLOADS[args.workload]
    config = {"workload": args.workload, "l2": "flushed before every step (256 MiB write, outside the events)",
              "parallelism": f"replicas x{world} (independent problems per rank)", "format": fmt,
              "shape": shape, "text": text}

    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, world, config)
        return

    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    iq.load_library()
    wl = Workload(args.workload, dev, peaks)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        flush.zero_()
        wl.step()
    torch.cuda.synchronize()

    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    dom_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with Clocks(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.zero_()
            step_ev[i][0].record()
            wl.step(dom_ev[i])
            step_ev[i][1].record()
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    iq.raise_for_flags(wl.flags)  # the timed steps' findings (none on these inputs)
    step_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in step_ev), dist, dev)
    dom_ms = [s.elapsed_time(e) for s, e in dom_ev]
    ms_per_step = step_ms / args.steps
    value = weak_scaling_value(wl.units, world, ms_per_step)

    # end to end through the public API from pinned host memory (same stream, events)
    host, h2d, d2h = wl.host_buffers()
    for _ in range(2):
        wl.e2e_step(host)
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(e2e_steps):
        wl.e2e_step(host)
    e.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(s.elapsed_time(e) / e2e_steps, dist, dev)
    e2e_value = weak_scaling_value(wl.units, world, e2e_ms)

    dec = decode_roofline(wl, dev, peaks) if rank == 0 else None
    fp32 = measure_fp32(dev, kinds=("ffma", "ffma2"), reps=3) if rank == 0 and wl.kind != "decode" else None
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    clocks = clk.summary()
    dom_avg = statistics.mean(dom_ms)
    traffic, tnote = kernel_traffic(wl.dominant, args.workload, wl.nblocks)
    if wl.kind == "decode":
        nbytes = wl.nblocks * (iq.BLOCK_BYTES[wl.fmt] + 512)
        gbs = nbytes / (dom_avg / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": wl.dominant, "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
                "traffic_source": tnote, "bytes_per_launch": nbytes, "ms_per_launch": round(dom_avg, 4)}
    else:
        achieved = wl.ops_per_launch / (dom_avg / 1e3) / 1e12
        peak = max(fp32.values())
        nominal = alu_peak_tops(peaks["sm_max_mhz"])
        roof = {"bound": "alu", "kernel": wl.dominant, "achieved": round(achieved, 3), "peak": peak,
                "unit": "Top/s", "frac": round(achieved / peak, 4), "traffic": traffic, "traffic_source": tnote,
                "ops_per_launch": wl.ops_per_launch, "ops_count": "algorithmic work (every candidate of the "
                "exhaustive search counts; fma and min one op each)", "ms_per_launch": round(dom_avg, 4),
                "peak_basis": "measured in this run: FP32 lane ops/s of iq_probe_fp32 (8 CTAs x 256 threads per "
                f"SM), the larger of scalar fma {fp32['ffma']} and packed fma.f32x2 {fp32['ffma2']} Top/s",
                "peak_nominal": round(nominal, 3), "frac_of_nominal": round(achieved / nominal, 4)}
        if wl.kind == "choice":
            roof["ops_executed_note"] = ("the count includes a gradient update after every group step; the "
                                         "kernel updates only after a switch")

    cpu = None
    if not args.no_cpu_baseline:
        rate, rows, cols, dt, cores, _ = oracle_sample_rate(args.workload, budget_s=12.0)
        cpu = {"value": round(rate, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"first {rows} rows x {cols} cols of the workload, encode + decode, {dt:.1f} s wall"}

    metric = "IQ decode Mweights/s" if wl.kind == "decode" else METRIC
    line = {"metric": metric, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config,
            "roofline": roof, "decode": dec, "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": ("public API calls on 16 pieces of the leading dimension, host-to-device copies, "
                            "kernels and device-to-host copies on three streams" if wl.kind == "encode" else
                            "public API calls, copies and kernels in order on one stream")},
            "gpu_launches": wl.launches_per_step * args.steps, "clocks": clocks,
            "peaks": {"source": peaks["source"], "hbm_gbs": peaks["hbm_gbs"]}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
