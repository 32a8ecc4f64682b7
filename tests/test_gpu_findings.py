"""Device-side findings through the C ABI (needs a B200): what a call returns and writes when the
data is bad, with and without a caller-owned flags word.

- With a flags word the calls stay asynchronous and the word holds the findings.
- Without one (flags == NULL in C) the call synchronises and returns the finding as a status, so
  bad data never comes back as IQ_OK.
- The choice search zeroes the payload of a row-block with a finding, reports picks 0 and a NaN
  objective, exactly as the oracle does, and leaves every other row-block as it is.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq
import oracle
from ggml_iq_codebook_b200 import build, synth

pytestmark = pytest.mark.gpu

IQ_ENONFINITE, IQ_EIMPORTANCE, IQ_EGRID = 5, 6, 9


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    iq.load_library()
    return torch.device("cuda:0")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_encode_without_flags_word_returns_the_finding(dev, grids, anchors):
    lib = iq.load_library()
    g = torch.from_numpy(grids["iq1_s"]).to(dev)
    desc = iq.make_desc("iq1_s", g, anchors["iq1_s"])
    w = synth.normal_bf16((4, 512), 0.02, 901).to(dev)
    imp = synth.lognormal((512,), 902).to(dev)
    out = torch.empty((4, 2, 50), dtype=torch.uint8, device=dev)

    def call(wt, it):
        return lib.iq_encode(ctypes.byref(desc), wt.data_ptr(), 0, 1, 4, 512, 512, 0, it.data_ptr(), 0, None, None,
                             0, 0, out.data_ptr(), None, _stream())

    assert call(w, imp) == 0
    w_bad = w.clone()
    w_bad[2, 7] = float("nan")
    assert call(w_bad, imp) == IQ_ENONFINITE
    assert not out[2, 0].any() and out[2, 1].any()      # the tainted block is zeroed, the others kept
    imp_bad = imp.clone()
    imp_bad[300] = -1.0
    assert call(w, imp_bad) == IQ_EIMPORTANCE
    g_bad = grids["iq1_s"].copy()
    g_bad[9, 1] = 3
    desc_bad = iq.make_desc("iq1_s", torch.from_numpy(g_bad).to(dev), anchors["iq1_s"])
    st = lib.iq_encode(ctypes.byref(desc_bad), w.data_ptr(), 0, 1, 4, 512, 512, 0, imp.data_ptr(), 0, None, None,
                       0, 0, out.data_ptr(), None, _stream())
    assert st == IQ_EGRID
    assert lib.iq_status_string(st).startswith(b"a grid value")


def _choice_inputs(fmt, grids, anchors, dev, rows=20, nblk=2, seed=911, std=0.02):
    base = "iq2_xs" if fmt == "g8" else fmt
    w = synth.normal_bf16((rows, 256 * nblk), std, seed)
    hess = torch.stack([synth.block_hessian(seed + 10 + b, offdiag_std=0.3) for b in range(nblk)])
    imp = oracle.sqrt_diag(hess.numpy())
    cand, _ = oracle.encode(base, grids[base], anchors[base], w, importance=imp, every_choice=True)
    return base, w, hess, cand


def _gpu_search(fmt, base, desc, w, hess, cand, dev):
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    obj = torch.empty((w.shape[0], w.shape[1] // 256), dtype=torch.float32, device=dev)
    cd = torch.from_numpy(cand).to(dev)
    if fmt == "g8":
        picks = iq.iq_choice_search_g8(desc, w.to(dev), hess.to(dev), cd, flags=flags, objective=obj)
        pay = None
    else:
        picks, pay = iq.iq_choice_search(desc, w.to(dev), hess.to(dev), cd, flags=flags, objective=obj)
        pay = pay.cpu().numpy()
    torch.cuda.synchronize()
    return picks.cpu().numpy(), pay, obj.cpu().numpy(), int(flags.item())


def _oracle_search(fmt, base, grid, w, hess, cand):
    if fmt == "g8":
        picks, obj, f = oracle.choice_search_g8(grid, w, hess.numpy(), cand, objective=True, return_flags=True)
        return picks, None, obj, f
    return oracle.choice_search(fmt, grid, w, hess.numpy(), cand, objective=True, return_flags=True)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m", "g8"])
def test_choice_search_findings_match_the_oracle(dev, grids, anchors, fmt):
    base, w, hess, cand = _choice_inputs(fmt, grids, anchors, dev)
    desc = iq.make_desc(base, torch.from_numpy(grids[base]).to(dev), anchors[base])
    w_bad = w.clone()
    w_bad[3, 40] = float("nan")                   # row 3, block 0
    w_bad[17, 511] = float("-inf")                # row 17, block 1
    h_bad = hess.clone()
    h_bad[1, 200, 3] = float("nan")               # block 1 of every row
    for wi, hi, want_flags in ((w, hess, 0), (w_bad, hess, iq.FLAG_NONFINITE), (w, h_bad, iq.FLAG_NONFINITE),
                               (w_bad, h_bad, iq.FLAG_NONFINITE)):
        got = _gpu_search(fmt, base, desc, wi, hi, cand, dev)
        want = _oracle_search(fmt, base, grids[base], wi, hi, cand)
        assert got[3] == want[3] == want_flags
        assert np.array_equal(got[0], want[0])
        if got[1] is not None:
            assert np.array_equal(got[1], want[1])
        assert np.array_equal(got[2].view(np.uint32), want[2].view(np.uint32))
    g_bad = grids[base].copy()
    g_bad[4, 0] = 2 if base != "iq1_s" and base != "iq1_m" else 5
    desc_bad = iq.make_desc(base, torch.from_numpy(g_bad).to(dev), anchors[base])
    got = _gpu_search(fmt, base, desc_bad, w, hess, cand, dev)
    want = _oracle_search(fmt, base, g_bad, w, hess, cand)
    assert got[3] == want[3] == iq.FLAG_GRID
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[2].view(np.uint32), want[2].view(np.uint32))
    if got[1] is not None:
        assert not got[1].any()


def test_choice_search_without_flags_word_raises(dev, grids, anchors):
    base, w, hess, cand = _choice_inputs("iq2_xs", grids, anchors, dev, rows=4, nblk=1)
    desc = iq.make_desc(base, torch.from_numpy(grids[base]).to(dev), anchors[base])
    cd = torch.from_numpy(cand).to(dev)
    iq.iq_choice_search(desc, w.to(dev), hess.to(dev), cd)   # finite data: no error
    h_bad = hess.clone()
    h_bad[0, 5, 5] = float("inf")
    with pytest.raises(iq.IQError, match="status 5"):
        iq.iq_choice_search(desc, w.to(dev), h_bad.to(dev), cd)


def test_choice_search_refuses_ragged_width(dev, grids, anchors):
    desc = iq.make_desc("iq2_xs", torch.from_numpy(grids["iq2_xs"]).to(dev), anchors["iq2_xs"])
    w = torch.zeros((4, 384), dtype=torch.bfloat16, device=dev)
    hess = torch.zeros((1, 256, 256), dtype=torch.float32, device=dev)
    cand = torch.zeros((16, 4, 1, 74), dtype=torch.uint8, device=dev)
    with pytest.raises(iq.IQError, match="multiple of 256"):
        iq.iq_choice_search(desc, w, hess, cand)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s"])
def test_choice_search_overflowing_gradient_is_not_a_finding(dev, grids, anchors, fmt):
    """A finite H whose products overflow fp32: the kernel's finiteness proof through the initial
    gradient fails, its exact scan of H finds every entry finite, so nothing is flagged, and picks,
    payload and objective still equal the oracle's (objective NaNs compared as NaN: their bit
    patterns are the hardware's)."""
    # unit-scale weights, so that H x Delta overflows once H sits near the top of the range
    base, w, hess, cand = _choice_inputs(fmt, grids, anchors, dev, rows=12, nblk=2, seed=933, std=1.0)
    desc = iq.make_desc(base, torch.from_numpy(grids[base]).to(dev), anchors[base])
    big = hess.clone()
    big[1] = big[1] * (3.0e38 / float(big[1].abs().max()))   # block 1 at the top of the fp32 range
    assert torch.isfinite(big).all()
    got = _gpu_search(fmt, base, desc, w, big, cand, dev)
    want = _oracle_search(fmt, base, grids[base], w, big, cand)
    assert got[3] == want[3] == 0
    assert np.array_equal(got[0], want[0])
    assert np.array_equal(got[1], want[1])
    g_obj, w_obj = got[2], want[2]
    assert np.array_equal(np.isnan(g_obj), np.isnan(w_obj))
    ok = ~np.isnan(w_obj)
    assert np.array_equal(g_obj[ok].view(np.uint32), w_obj[ok].view(np.uint32))
    assert not np.isfinite(w_obj[:, 1]).all() and np.isfinite(w_obj[:, 0]).all()  # block 1 overflows
