"""Every row of the five full-size workloads against the CPU oracle (needs a B200).

The oracle's outputs at these sizes were hashed row by row by tests/golden/make_digests.py (which
calls only the oracle and the seeded generator); here the GPU runs each workload in the launch
configuration bench.py times (one call per kernel over the whole weight, or over all 256 experts),
and every row of its output is hashed the same way and compared. A mismatch names the first rows
that differ.
"""

from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq
from ggml_iq_codebook_b200 import build, synth

from golden.make_digests import row_digests

pytestmark = pytest.mark.gpu

DIGESTS = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "digests")


def _want(name):
    meta = json.load(open(os.path.join(DIGESTS, f"{name}.json")))
    z = np.load(os.path.join(DIGESTS, f"{name}.npz"))
    return {k: z[k] for k in meta["arrays"]}


def _compare(name, what, got, want):
    assert got.shape == want.shape, (name, what, got.shape, want.shape)
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{name} {what}: {len(bad)} rows differ, first {bad[:8].tolist()}"


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    iq.load_library()
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def descs(dev, grids, anchors):
    return {fmt: iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
            for fmt in ("iq1_s", "iq2_xs")}


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name,make", [
    ("iq1s_64x256", synth.workload_iq1s_64x256),
    ("iq1s_4096x4096_weighted", synth.workload_iq1s_4096x4096_weighted),
    ("iq2xs_8192x4096", synth.workload_iq2xs_8192x4096),
])
def test_every_row_encode_decode(dev, descs, name, make):
    wl = make()
    imp = None if wl["importance"] is None else wl["importance"].to(dev)
    pay = iq.iq_encode(descs[wl["fmt"]], wl["w"].to(dev), imp)
    dec = iq.iq_decode(descs[wl["fmt"]], pay, torch.bfloat16)
    want = _want(name)
    _compare(name, "payload", row_digests(pay.cpu().numpy()), want["payload"])
    _compare(name, "bf16 decode", row_digests(_bits(dec).reshape(dec.shape[0], -1)), want["decode_bf16"])


def test_every_row_moe_256x1536x4096_one_call(dev, descs):
    name = "iq1s_moe_256x1536x4096"
    if not os.path.exists(os.path.join(DIGESTS, f"{name}.npz")):
        pytest.fail("the MoE digests are missing: run tests/golden/make_digests.py")
    wl = synth.workload_iq1s_moe(device=dev)
    pay = iq.iq_encode(descs["iq1_s"], wl["w"], wl["importance"].to(dev))
    del wl
    dec = iq.iq_decode(descs["iq1_s"], pay, torch.bfloat16)
    want = _want(name)
    got_p = pay.cpu().numpy()
    got_d = _bits(dec)
    del pay, dec
    torch.cuda.empty_cache()
    e, r = want["payload"].shape
    _compare(name, "payload", row_digests(got_p.reshape(e * r, -1)).reshape(e, r), want["payload"])
    _compare(name, "bf16 decode", row_digests(got_d.reshape(e * r, -1)).reshape(e, r), want["decode_bf16"])


def test_every_row_choice_search_4096x4096(dev, descs):
    name = "choice_iq2xs_4096x4096"
    wl = synth.workload_choice_iq2xs()
    wd, hd = wl["w"].to(dev), wl["hess"].to(dev)
    cand = iq.iq_encode(descs["iq2_xs"], wd, iq.iq_sqrt_diag(hd), every_choice=True)
    obj = torch.empty((wd.shape[0], wd.shape[1] // 256), dtype=torch.float32, device=dev)
    picks, pay = iq.iq_choice_search(descs["iq2_xs"], wd, hd, cand, objective=obj)
    want = _want(name)
    _compare(name, "candidates", row_digests(np.moveaxis(cand.cpu().numpy(), 0, 1)), want["candidates"])
    _compare(name, "picks", row_digests(picks.cpu().numpy()), want["picks"])
    _compare(name, "payload", row_digests(pay.cpu().numpy()), want["payload"])
    _compare(name, "objective", row_digests(obj.cpu().numpy().view(np.uint32)), want["objective"])
