"""The per-block calibration loop on the GPU against the CPU oracle, bit for bit (needs a B200).

One call runs every block of a weight in order: the every-choice encode of the compensated
weights, the local-Hessian choice search, and GPTQ's propagation of the block's error to the later
columns. Payloads, picks and the compensated weights each block was quantised from must equal
the oracle's exactly, for every format, on shapes that span several update tiles and a ragged
row tail.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq
import oracle
from ggml_iq_codebook_b200 import build, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    iq.load_library()
    return torch.device("cuda:0")


def _inputs(rows, nblk, seed, cross_std=0.05):
    w = synth.normal_bf16((rows, 256 * nblk), 0.02, seed)
    U = synth.inverse_hessian_factor(nblk, seed=seed + 100, cross_seed=seed + 200, cross_std=cross_std)
    hess = torch.stack([synth.block_hessian(seed + 100 + b) for b in range(nblk)])
    return w, U, hess


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
@pytest.mark.parametrize("rows,nblk", [(40, 3), (137, 2)])
def test_loop_matches_the_oracle(dev, grids, anchors, fmt, rows, nblk):
    if fmt == "iq1_s" and rows > 40:
        rows = 37  # the IQ1_S oracle is the slow one
    w, U, hess = _inputs(rows, nblk, 400 + rows)
    desc = iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    pay, picks, w_work = iq.iq_gptq_blocks(desc, w.to(dev), hess.to(dev), U.to(dev), flags=flags)
    torch.cuda.synchronize()
    want_pay, want_picks, want_w, want_flags = oracle.gptq_blocks(fmt, grids[fmt], anchors[fmt], w, hess.numpy(),
                                                                  U.numpy())
    assert int(flags.item()) == want_flags == 0
    assert np.array_equal(w_work.cpu().numpy().view(np.uint32), want_w.view(np.uint32))
    assert np.array_equal(picks.cpu().numpy(), want_picks)
    assert np.array_equal(pay.cpu().numpy(), want_pay)
    assert not np.array_equal(want_w, w.float().numpy())  # the later blocks were compensated


def test_wide_weight_spans_update_tiles(dev, grids, anchors):
    """1024 columns (three update launches of 768, 512 and 256 columns) over 300 rows (three row
    tiles, the last ragged)."""
    fmt = "iq2_xs"
    w, U, hess = _inputs(300, 4, 431)
    desc = iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
    pay, picks, w_work = iq.iq_gptq_blocks(desc, w.to(dev), hess.to(dev), U.to(dev))
    want_pay, want_picks, want_w, _ = oracle.gptq_blocks(fmt, grids[fmt], anchors[fmt], w, hess.numpy(), U.numpy())
    assert np.array_equal(w_work.cpu().numpy().view(np.uint32), want_w.view(np.uint32))
    assert np.array_equal(picks.cpu().numpy(), want_picks) and np.array_equal(pay.cpu().numpy(), want_pay)


def test_one_block_is_the_plain_pipeline(dev, grids, anchors):
    """A single block has nothing to propagate: the loop is the every-choice encode plus the
    choice search of the weight itself."""
    fmt = "iq2_xs"
    w, U, hess = _inputs(50, 1, 441)
    desc = iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
    wd, hd = w.to(dev), hess.to(dev)
    pay, picks, w_work = iq.iq_gptq_blocks(desc, wd, hd, U.to(dev))
    cand = iq.iq_encode(desc, wd, iq.iq_sqrt_diag(hd), every_choice=True)
    want_picks, want_pay = iq.iq_choice_search(desc, wd, hd, cand)
    assert torch.equal(picks, want_picks) and torch.equal(pay, want_pay)
    assert torch.equal(w_work, wd.float())


def test_findings_without_flags_word(dev, grids, anchors):
    fmt = "iq2_xs"
    w, U, hess = _inputs(8, 2, 451)
    desc = iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
    w_bad = w.clone()
    w_bad[2, 3] = float("nan")
    with pytest.raises(iq.IQError, match="status 5"):
        iq.iq_gptq_blocks(desc, w_bad.to(dev), hess.to(dev), U.to(dev))
    with pytest.raises(iq.IQError):  # a workspace one byte short is refused before any launch
        need = iq.iq_gptq_workspace_bytes(fmt, 8)
        iq.iq_gptq_blocks(desc, w.to(dev), hess.to(dev), U.to(dev),
                          workspace=torch.empty(need - 1, dtype=torch.uint8, device=dev))
