#!/usr/bin/env python
"""Write per-row digests of the CPU oracle's outputs on the five full-size workloads.

The GPU parity test (tests/test_gpu_full_parity.py) hashes every row of the library's output at
these sizes and compares it with the digests stored here, so that every row of every workload is
checked against bytes the GPU path did not produce, without running the oracle for hours inside
the test. This script calls only the oracle (oracle/) and the seeded input generator (synth.py).

A row digest is the first 4 bytes (little endian) of BLAKE2b over that row's bytes:
  encode workloads   payload [rows, cols/256, B] and the bf16 decode [rows, cols] of that payload
  MoE batch          the same per (expert, row)
  choice search      the every-choice candidates [16, rows, nblk, 74] taken per row (all 16
                     choices), the picks [rows, nblk, 16], the payload [rows, nblk, 74] and the
                     objective [rows, nblk] (fp32 bits)

The oracle is compiled once more with -O3 -march=native (IEEE semantics unchanged: still
-ffp-contract=off and no fast-math). Before anything is written, the first rows of each workload
are encoded by both builds and must agree byte for byte.

    python tests/golden/make_digests.py [--only NAME ...] [--scratch DIR] [--threads N]

The MoE batch (1.6 G weights) takes about two hours on 8 cores; its per-expert results are kept in
--scratch so that an interrupted run resumes where it stopped.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import tempfile
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from ggml_iq_codebook_b200 import synth  # noqa: E402

OUT_DIR = os.path.join(HERE, "digests")
ANCHOR = {"iq1_s": 0.61, "iq2_xs": 0.9}  # the library's default anchors (IQ1_S's is #2450's)


def row_digests(a: np.ndarray) -> np.ndarray:
    """uint32 digest of each leading-axis row of `a`."""
    a = np.ascontiguousarray(a)
    flat = a.reshape(a.shape[0], -1).view(np.uint8)
    out = np.empty(a.shape[0], dtype=np.uint32)
    for r in range(a.shape[0]):
        out[r] = int.from_bytes(hashlib.blake2b(flat[r].tobytes(), digest_size=4).digest(), "little")
    return out


def bf16_decode(fmt, grid, payload) -> np.ndarray:
    """The oracle's exact fp32 decode rounded to bf16 (RNE), as uint16 bits [rows, cols]."""
    y = oracle.decode(fmt, grid, payload)  # [rows, nblk, 256]
    return oracle.f32_to_bf16_bits(y.reshape(y.shape[0], -1))


def check_builds(fmt, grid, w, imp, rows=2):
    """The optimised build must reproduce the plain build's payload on the first rows."""
    with oracle.library(oracle.build()):
        want, _ = oracle.encode(fmt, grid, ANCHOR[fmt], w[:rows], importance=imp)
    got, _ = oracle.encode(fmt, grid, ANCHOR[fmt], w[:rows], importance=imp)
    if not np.array_equal(got, want):
        raise SystemExit(f"optimised oracle build differs from the plain build ({fmt})")


def encode_rows(fmt, grid, w, imp, chunk=256):
    rows = w.shape[0]
    pay = []
    for r0 in range(0, rows, chunk):
        p, flags = oracle.encode(fmt, grid, ANCHOR[fmt], w[r0:r0 + chunk], importance=imp)
        if flags:
            raise SystemExit(f"oracle flagged the workload input (flags {flags})")
        pay.append(p)
    return np.concatenate(pay)


def dense(name, wl, grid):
    fmt, w, imp = wl["fmt"], wl["w"], wl["importance"]
    imp = None if imp is None else imp.numpy()
    check_builds(fmt, grid, w, imp)
    pay = encode_rows(fmt, grid, w, imp)
    return {"payload": row_digests(pay), "decode_bf16": row_digests(bf16_decode(fmt, grid, pay))}


def moe(scratch, experts=256, rows=1536, cols=4096):
    grid = synth.iq1s_grid()
    imp = synth.lognormal((experts, cols), 3004).numpy()
    os.makedirs(scratch, exist_ok=True)
    check_builds("iq1_s", grid, synth.expert_bf16(0, rows, cols, 0.02, 1004), imp[0])
    pay_d, dec_d = [], []
    t0 = time.time()
    for e in range(experts):
        path = os.path.join(scratch, f"moe_expert_{e:03d}.npz")
        if not os.path.exists(path):
            w = synth.expert_bf16(e, rows, cols, 0.02, 1004)
            pay = encode_rows("iq1_s", grid, w, imp[e])
            np.savez(path + ".tmp.npz", payload=row_digests(pay),
                     decode_bf16=row_digests(bf16_decode("iq1_s", grid, pay)))
            os.replace(path + ".tmp.npz", path)
            print(f"  expert {e}: {time.time() - t0:.0f} s", flush=True)
        z = np.load(path)
        pay_d.append(z["payload"])
        dec_d.append(z["decode_bf16"])
    return {"payload": np.stack(pay_d), "decode_bf16": np.stack(dec_d)}


def choice():
    wl = synth.workload_choice_iq2xs()
    grid = synth.iq2xs_grid()
    w, hess = wl["w"], wl["hess"].numpy()
    imp = oracle.sqrt_diag(hess)
    check_builds("iq2_xs", grid, w, imp)
    cand = []
    for r0 in range(0, w.shape[0], 256):
        c, flags = oracle.encode("iq2_xs", grid, ANCHOR["iq2_xs"], w[r0:r0 + 256], importance=imp, every_choice=True)
        if flags:
            raise SystemExit(f"oracle flagged the workload input (flags {flags})")
        cand.append(c)
    cand = np.concatenate(cand, axis=1)  # [16, rows, nblk, 74]
    picks, pay, obj = oracle.choice_search("iq2_xs", grid, w, hess, cand, objective=True)
    return {"candidates": row_digests(np.moveaxis(cand, 0, 1)), "picks": row_digests(picks),
            "payload": row_digests(pay), "objective": row_digests(obj.view(np.uint32))}


JOBS = {
    "iq1s_64x256": lambda a: dense("iq1s_64x256", synth.workload_iq1s_64x256(), synth.iq1s_grid()),
    "iq1s_4096x4096_weighted": lambda a: dense("iq1s_4096x4096_weighted", synth.workload_iq1s_4096x4096_weighted(),
                                               synth.iq1s_grid()),
    "iq2xs_8192x4096": lambda a: dense("iq2xs_8192x4096", synth.workload_iq2xs_8192x4096(), synth.iq2xs_grid()),
    "choice_iq2xs_4096x4096": lambda a: choice(),
    "iq1s_moe_256x1536x4096": lambda a: moe(a.scratch),
}

RECIPES = {
    "iq1s_64x256": "synth.workload_iq1s_64x256: [64, 256] N(0, 0.02^2) seed 1001, uniform importance",
    "iq1s_4096x4096_weighted": "synth.workload_iq1s_4096x4096_weighted: [4096, 4096] N(0, 0.02^2) seed 1002, 41 "
                               "columns (seed 2002) x8, importance sqrt(lognormal) seed 3002",
    "iq2xs_8192x4096": "synth.workload_iq2xs_8192x4096: [8192, 4096] N(0, 0.015^2) seed 1003, importance "
                       "lognormal seed 3003",
    "choice_iq2xs_4096x4096": "synth.workload_choice_iq2xs: [4096, 4096] N(0, 0.02^2) seed 1005, H blocks seeds "
                              "5000..5015; candidates = IQ2_XS every-choice encode under sqrt(diag H)",
    "iq1s_moe_256x1536x4096": "synth.workload_iq1s_moe: 256 x [1536, 4096] N(0, 0.02^2), expert e seed "
                              "1004 * 1024 + e, importance lognormal [256, 4096] seed 3004",
}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", nargs="*", default=None)
    ap.add_argument("--scratch", default=os.path.join(tempfile.gettempdir(), "iq_digest_scratch"))
    ap.add_argument("--threads", type=int, default=os.cpu_count())
    args = ap.parse_args()
    oracle._load(oracle.build_optimised())
    oracle.set_threads(args.threads)
    src_sha = hashlib.sha256(open(os.path.join(ROOT, "oracle", "iq_oracle.c"), "rb").read()).hexdigest()
    os.makedirs(OUT_DIR, exist_ok=True)
    for name in (args.only or list(JOBS)):
        t0 = time.time()
        print(f"{name} ...", flush=True)
        arrays = JOBS[name](args)
        np.savez_compressed(os.path.join(OUT_DIR, f"{name}.npz"), **arrays)
        meta = {"workload": name, "recipe": RECIPES[name], "digest": "blake2b, first 4 bytes little endian, per row",
                "arrays": {k: list(v.shape) for k, v in arrays.items()}, "oracle_source_sha256": src_sha,
                "oracle_build": "gcc -O3 -march=native -ffp-contract=off -fno-fast-math (checked against -O2)",
                "seconds": round(time.time() - t0, 1)}
        with open(os.path.join(OUT_DIR, f"{name}.json"), "w") as f:
            json.dump(meta, f, indent=1)
            f.write("\n")
        print(f"{name}: {meta['seconds']} s", flush=True)


if __name__ == "__main__":
    main()
