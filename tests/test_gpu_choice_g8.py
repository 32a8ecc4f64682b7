"""The choice search with eight candidates per 8-weight group: CUDA path vs the oracle, bit for bit.

32 groups of 8 columns per block, each choosing among the IQ2_XS every-choice decodes for
ls = 8..15 (PR #3158's steps). Picks and objectives over ragged row counts (16 rows per CTA),
several CTAs and blocks, an expert stack, a strided single-block view, and the 4096 x 4096
launch the benchmark times, checked on sampled rows.
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


@pytest.fixture(scope="module")
def desc(dev, grids, anchors):
    return iq.make_desc("iq2_xs", torch.from_numpy(grids["iq2_xs"]).to(dev), anchors["iq2_xs"])


def _case(rows, nblk, seed, offdiag=0.3):
    w = synth.normal_bf16((rows, nblk * 256), 0.02, seed)
    hess = torch.stack([synth.block_hessian(seed + 10 + b, offdiag_std=offdiag) for b in range(nblk)])
    return w, hess


def _oracle(grids, anchors, w, hess):
    imp = oracle.sqrt_diag(hess.numpy())
    cand, _ = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, importance=imp, every_choice=True)
    return cand, oracle.choice_search_g8(grids["iq2_xs"], w, hess.numpy(), cand, objective=True)


@pytest.mark.parametrize("rows,nblk,offdiag", [(1, 1, 0.3), (13, 2, 0.3), (37, 3, 0.02), (40, 2, 0.3)])
def test_picks_and_objective_match_oracle(dev, desc, grids, anchors, rows, nblk, offdiag):
    w, hess = _case(rows, nblk, 400 + rows, offdiag)
    hd = hess.to(dev)
    cand_d = iq.iq_encode(desc, w.to(dev), iq.iq_sqrt_diag(hd), every_choice=True)
    obj = torch.empty((rows, nblk), dtype=torch.float32, device=dev)
    picks = iq.iq_choice_search_g8(desc, w.to(dev), hd, cand_d, objective=obj)
    torch.cuda.synchronize()
    cand, (want_p, want_obj) = _oracle(grids, anchors, w, hess)
    assert np.array_equal(cand_d.cpu().numpy(), cand)
    got = picks.cpu().numpy()
    assert got.shape == (rows, nblk, 32) and got.min() >= 8 and got.max() < 16
    assert np.array_equal(got, want_p)
    assert np.array_equal(obj.cpu().numpy().view(np.uint32), want_obj.view(np.uint32))


def test_expert_stack_in_one_launch(dev, desc, grids, anchors):
    nexp, rows, nblk = 3, 5, 2
    w = synth.normal_bf16((nexp, rows, nblk * 256), 0.02, 420)
    hess = torch.stack([torch.stack([synth.block_hessian(430 + 10 * e + b, offdiag_std=0.3) for b in range(nblk)])
                        for e in range(nexp)])
    hd = hess.to(dev)
    imp_d = iq.iq_sqrt_diag(hd.reshape(-1, 256, 256)).reshape(nexp, nblk * 256)
    cand_d = iq.iq_encode(desc, w.to(dev), imp_d, every_choice=True)
    picks = iq.iq_choice_search_g8(desc, w.to(dev), hd, cand_d).cpu().numpy()
    imp = oracle.sqrt_diag(hess.numpy()).reshape(nexp, nblk * 256)
    cand = np.stack([oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w[e], importance=imp[e],
                                   every_choice=True)[0] for e in range(nexp)], axis=1)
    assert np.array_equal(cand_d.cpu().numpy(), cand)
    (want,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess.numpy(), cand)
    assert np.array_equal(picks, want)


def test_one_block_of_a_wider_weight(dev, desc, grids, anchors):
    """A view of block 1 of a 3-block weight with its candidate slices: strided rows and cand."""
    rows, nblk = 21, 3
    w, hess = _case(rows, nblk, 440)
    hd = hess.to(dev)
    wd = w.to(dev)
    cand_d = iq.iq_encode(desc, wd, iq.iq_sqrt_diag(hd), every_choice=True)
    got = iq.iq_choice_search_g8(desc, wd[:, 256:512], hd[1:2], cand_d[:, :, 1:2]).cpu().numpy()
    cand, (want, _) = _oracle(grids, anchors, w, hess)
    assert np.array_equal(got[:, 0], want[:, 1])


def test_rejects_other_formats(dev, grids, anchors):
    d1 = iq.make_desc("iq1_s", torch.from_numpy(grids["iq1_s"]).to(dev), anchors["iq1_s"])
    w, hess = _case(2, 1, 450)
    cand = torch.zeros((16, 2, 1, 50), dtype=torch.uint8, device=dev)
    with pytest.raises(iq.IQError):
        iq.iq_choice_search_g8(d1, w.to(dev), hess.to(dev), cand)


def test_full_size_launch_on_sampled_rows(dev, desc, grids, anchors):
    """The 4096 x 4096 workload in one launch (4096 rows x 16 blocks); the oracle recomputes sampled
    rows, each row's search depending on that row alone."""
    wl = synth.workload_choice_iq2xs()
    w, hess = wl["w"], wl["hess"]
    hd = hess.to(dev)
    cand_d = iq.iq_encode(desc, w.to(dev), iq.iq_sqrt_diag(hd), every_choice=True)
    obj = torch.empty((w.shape[0], w.shape[1] // 256), dtype=torch.float32, device=dev)
    picks = iq.iq_choice_search_g8(desc, w.to(dev), hd, cand_d, objective=obj).cpu().numpy()
    obj = obj.cpu().numpy()
    rows = np.sort(np.random.default_rng(460).choice(w.shape[0], 4, replace=False))
    imp = oracle.sqrt_diag(hess.numpy())
    cand, _ = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w[rows], importance=imp, every_choice=True)
    want_p, want_obj = oracle.choice_search_g8(grids["iq2_xs"], w[rows], hess.numpy(), cand, objective=True)
    assert np.array_equal(picks[rows], want_p)
    assert np.array_equal(obj[rows].view(np.uint32), want_obj.view(np.uint32))
