"""Pins of the oracle's per-block calibration loop (CPU only).

The loop ([#3218]: GPTQ with local_hessian_scales searches one block at a time) quantises a weight
one 256-column block after the other: every-choice encode under sqrt(diag H_b), local-Hessian
choice search under H_b, then GPTQ's propagation of the block's error to the later columns
(Frantar et al. 2022): W[:, rest] -= (E U_bb^-1) U_b,rest with H^-1 = U^T U.

- The propagation formula itself is checked against the optimum it claims, in fp64: with delta the
  amount taken off the later columns, the error left on the trailing columns is [E, delta], and
  for the trailing Hessian A = H[>= b, >= b] delta minimises [E, delta] A [E, delta]^T.
- The oracle's fp32 loop is replayed in fp64 from its own payloads: the weights each block was
  quantised from must follow the formula within fp32 rounding.
- With no coupling between blocks (U block-diagonal) the loop is the plain per-block pipeline.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from ggml_iq_codebook_b200 import synth


def _inputs(rows, nblk, seed, cross_std=0.02):
    w = synth.normal_bf16((rows, 256 * nblk), 0.02, seed)
    U = synth.inverse_hessian_factor(nblk, seed=seed + 100, cross_seed=seed + 200, cross_std=cross_std)
    hess = torch.stack([synth.block_hessian(seed + 100 + b) for b in range(nblk)]).numpy()
    return w, U.numpy(), hess


def test_propagation_is_the_obs_optimum():
    """GPTQ's closed form against the minimiser of the trailing quadratic (fp64)."""
    nblk = 3
    U = synth.inverse_hessian_factor(nblk, seed=11, cross_seed=12, cross_std=0.05).double().numpy()
    H = np.linalg.inv(U.T @ U)
    rng = np.random.default_rng(13)
    for b in range(nblk - 1):
        s, r = slice(256 * b, 256 * (b + 1)), slice(256 * (b + 1), None)
        E = rng.normal(size=(4, 256))
        delta = (E @ np.linalg.inv(U[s, s])) @ U[s, r]          # the amount subtracted from W[:, rest]
        A = H[256 * b:, 256 * b:]
        Abr, Arr = A[:256, 256:], A[256:, 256:]
        # the error left is [E, d] (original minus compensated weights); minimise
        # [E, d] A [E, d]^T over d: d = -E Abr Arr^-1
        d_opt = -E @ Abr @ np.linalg.inv(Arr)
        assert np.allclose(delta, d_opt, rtol=1e-8, atol=1e-10)
        # and a sign or transposition slip is not the optimum
        assert not np.allclose(-delta, d_opt, atol=1e-6)
        assert not np.allclose((E @ np.linalg.inv(U[s, s]).T) @ U[s, r], d_opt, atol=1e-6)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s"])
def test_block_diagonal_factor_is_the_plain_pipeline(grids, anchors, fmt):
    rows, nblk = 3, 2
    w, U, hess = _inputs(rows, nblk, 301)
    for b in range(nblk):  # drop the coupling between blocks
        U[256 * b:256 * (b + 1), 256 * (b + 1):] = 0.0
    pay, picks, w_work, flags = oracle.gptq_blocks(fmt, grids[fmt], anchors[fmt], w, hess, U)
    assert flags == 0
    assert np.array_equal(w_work, w.float().numpy())
    imp = oracle.sqrt_diag(hess)
    cand, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    want_p, want_pay = oracle.choice_search(fmt, grids[fmt], w, hess, cand)
    assert np.array_equal(picks, want_p) and np.array_equal(pay, want_pay)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
def test_loop_replays_in_fp64(grids, anchors, fmt):
    """Each block was quantised from W - sum over earlier blocks of E U_bb^-1 U_b,later, with E the
    error of that block's own payload; and each block's payload is the one-block pipeline applied
    to the weights it was quantised from."""
    rows, nblk = (4, 3) if fmt != "iq1_s" else (2, 3)
    w, U, hess = _inputs(rows, nblk, 311, cross_std=0.05)
    pay, picks, w_work, flags = oracle.gptq_blocks(fmt, grids[fmt], anchors[fmt], w, hess, U)
    assert flags == 0
    Ud = U.astype(np.float64)
    q = oracle.decode(fmt, grids[fmt], pay).reshape(rows, -1).astype(np.float64)
    ref = w.double().numpy().copy()
    moved = 0.0
    for b in range(nblk):
        s = slice(256 * b, 256 * (b + 1))
        got = w_work[:, s].astype(np.float64)
        scale = np.abs(ref[:, s]).max()
        assert np.allclose(got, ref[:, s], rtol=0, atol=2e-5 * scale), (b, np.abs(got - ref[:, s]).max())
        moved = max(moved, np.abs(got - w.double().numpy()[:, s]).max())
        E = got - q[:, s]                                   # the error of the block's own payload
        ref[:, 256 * (b + 1):] -= (E @ np.linalg.inv(Ud[s, s])) @ Ud[s, 256 * (b + 1):]
        # block b's payload is the one-block pipeline on the weights it was quantised from
        imp = oracle.sqrt_diag(hess[b:b + 1])
        cand, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w_work[:, s], importance=imp, every_choice=True)
        want_p, want_pay = oracle.choice_search(fmt, grids[fmt], w_work[:, s], hess[b:b + 1], cand)
        assert np.array_equal(picks[:, b:b + 1], want_p) and np.array_equal(pay[:, b:b + 1], want_pay)
    assert moved > 1e-4  # the later blocks really were compensated
