"""Pins of the oracle's choice search with eight candidates per 8-weight group (CPU only).

The local-Hessian search of PR #3158 (steps unchanged) run over 32 groups of 8 columns, each
group choosing among the IQ2_XS every-choice decodes (PR #3159) for ls = 8..15. What fixes it:

* every decision of step 2 and of both sweeps replayed on the direct fp64 objective
  (x - xhat)^T H (x - xhat), and the sweeps do switch on correlated H;
* H block-diagonal over the 8-column groups makes the sweeps no-ops; H = I picks, per group, the
  least squared error among the eight candidates;
* the candidates for ls 0..7 are never read, the ones for 8..15 are;
* the reported objective is the final quadratic form, recomputed in fp64 from the picks;
* a stack of experts equals one call per expert with its own Hessians.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import replay_choice_search
from ggml_iq_codebook_b200 import synth

G, W, LS0 = 32, 8, 8


def _case(grids, anchors, rows, nblk, seed, offdiag):
    w = synth.normal_bf16((rows, nblk * 256), 0.02, seed)
    hess = torch.stack([synth.block_hessian(seed + 10 + b, offdiag_std=offdiag) for b in range(nblk)]).numpy()
    imp = oracle.sqrt_diag(hess)
    cand, flags = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, importance=imp, every_choice=True)
    assert flags == 0
    return w, hess, cand


def _deltas(grids, w, cand, r, b):
    """fp64 x - xhat for the eight candidates ls = 8..15 of row r, block b: [8, 256]."""
    x = w.double().numpy()[r, 256 * b:256 * b + 256]
    return x[None] - oracle.decode("iq2_xs", grids["iq2_xs"], cand[LS0:, r, b]).astype(np.float64)


def _assemble(dl, picks):
    return np.concatenate([dl[picks[g] - LS0, W * g:W * g + W] for g in range(G)])


@pytest.mark.parametrize("offdiag", [0.02, 0.3])
def test_decisions_replay_in_fp64(grids, anchors, offdiag):
    rows, nblk = 5, 2
    w, hess, cand = _case(grids, anchors, rows, nblk, 301, offdiag)
    picks, trace = oracle.choice_search_g8(grids["iq2_xs"], w, hess, cand, trace=True)
    assert picks.shape == (rows, nblk, G) and picks.min() >= LS0 and picks.max() < 16
    switches = 0
    for r in range(rows):
        for b in range(nblk):
            viol, sw, objs = replay_choice_search(_deltas(grids, w, cand, r, b), hess[b], G,
                                                  trace[r, b].astype(int) - LS0, rel_tol=3e-5)
            assert not viol, viol
            assert objs[2] <= objs[1] * (1 + 1e-6) and objs[1] <= objs[0] * (1 + 1e-6)
            assert np.array_equal(picks[r, b], trace[r, b, 2])
            switches += sw
    if offdiag > 0.1:
        assert switches > 0
    assert len(np.unique(picks)) >= 4


def test_block_diagonal_hessian_makes_sweeps_noops(grids, anchors):
    w, hess, cand = _case(grids, anchors, 3, 1, 311, 0.3)
    hb = hess * np.kron(np.eye(G), np.ones((W, W))).astype(np.float32)[None]
    _, trace = oracle.choice_search_g8(grids["iq2_xs"], w, hb, cand, trace=True)
    assert np.array_equal(trace[..., 0, :], trace[..., 1, :])
    assert np.array_equal(trace[..., 0, :], trace[..., 2, :])


def test_identity_hessian_picks_least_squared_error(grids, anchors):
    rows = 4
    w = synth.normal_bf16((rows, 256), 0.02, 321)
    cand, _ = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, every_choice=True)
    (picks,) = oracle.choice_search_g8(grids["iq2_xs"], w, np.eye(256, dtype=np.float32)[None], cand)
    for r in range(rows):
        dl = _deltas(grids, w, cand, r, 0)
        for g in range(G):
            err = (dl[:, W * g:W * g + W] ** 2).sum(1)
            got = err[picks[r, 0, g] - LS0]
            assert got <= err.min() * (1 + 1e-5), (r, g)


def test_reads_only_the_candidates_for_ls_8_to_15(grids, anchors):
    w, hess, cand = _case(grids, anchors, 4, 2, 331, 0.3)
    (picks,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess, cand)
    scrambled = cand.copy()
    scrambled[:LS0] = np.random.default_rng(332).integers(0, 256, scrambled[:LS0].shape, dtype=np.uint8)
    (again,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess, scrambled)
    assert np.array_equal(again, picks)
    swapped = cand.copy()
    swapped[[LS0, 15]] = cand[[15, LS0]]              # exchange the candidates for ls 8 and 15
    (other,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess, swapped)
    assert np.array_equal(np.where(other == 15, 8, np.where(other == 8, 15, other)), picks)


def test_objective_is_the_final_quadratic_form(grids, anchors):
    rows, nblk = 4, 2
    w, hess, cand = _case(grids, anchors, rows, nblk, 341, 0.3)
    picks, obj = oracle.choice_search_g8(grids["iq2_xs"], w, hess, cand, objective=True)
    assert picks.min() >= LS0 and picks.max() < 16
    for r in range(rows):
        for b in range(nblk):
            dl = _assemble(_deltas(grids, w, cand, r, b), picks[r, b])
            H = hess[b].astype(np.float64)
            scale = np.abs(dl) @ np.abs(H) @ np.abs(dl)
            assert abs(float(obj[r, b]) - dl @ H @ dl) <= 1e-5 * scale, (r, b)


def test_experts_use_their_own_hessians(grids, anchors):
    nexp, rows, nblk = 3, 3, 2
    w = synth.normal_bf16((nexp, rows, nblk * 256), 0.02, 351)
    hess = np.stack([np.stack([synth.block_hessian(360 + 10 * e + b, offdiag_std=0.3).numpy() for b in range(nblk)])
                     for e in range(nexp)])
    imp = oracle.sqrt_diag(hess).reshape(nexp, nblk * 256)
    cand = np.stack([oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w[e], importance=imp[e],
                                   every_choice=True)[0] for e in range(nexp)], axis=1)
    (picks,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess, cand)
    assert picks.shape == (nexp, rows, nblk, G)
    for e in range(nexp):
        (pe,) = oracle.choice_search_g8(grids["iq2_xs"], w[e], hess[e], cand[:, e])
        assert np.array_equal(picks[e], pe)
    (other,) = oracle.choice_search_g8(grids["iq2_xs"], w, hess[[1, 2, 0]], cand)
    assert not np.array_equal(other, picks)
