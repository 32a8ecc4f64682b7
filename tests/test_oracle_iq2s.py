"""Pins of the oracle's IQ2_S encoder and decoder (CPU only, no GPU).

IQ2_S (PR #2512 codec and PR #2565 CUDA encoder commit texts, on the page of PR #2525): a
1024-entry magnitude grid and eight sign bits for each group, so the encoder keeps the input's
signs and searches the magnitudes alone; a 4-bit local scale per 16 weights. What fixes it:

* a hand-built 82-byte block decoded against values written out from the layout reading;
* every sign mask equals the input's sign bits (no parity flip, unlike IQ2_XS);
* fp64 brute force: the picks reach the minimum of the direct residual over (ls, entry);
* ties to the lowest entry and the lowest ls, uniform-importance invariance, every-choice ==
  fixed choices, the zero and range policy, and the static-scale round trip.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import iq2s_fields, iq2xs_group_objectives, signs_of_mask
from ggml_iq_codebook_b200 import synth

ANCHOR = 0.9


def _case(rows, cols, seed, std=0.015):
    w = synth.normal_bf16((rows, cols), std, seed)
    w = synth.with_outlier_columns(w, synth.outlier_columns(cols, 0.05, seed + 1))
    return w, synth.lognormal((cols,), seed + 2)


def _enc(grids, w, **kw):
    return oracle.encode("iq2_s", grids["iq2_s"], ANCHOR, w, **kw)


def test_decode_hand_built_block():
    grid = np.ones((1024, 8), np.int8)
    grid[0x2C5] = [1, 3, 5, 7, 7, 5, 3, 1]
    grid[0x107] = [7, 7, 7, 7, 1, 1, 1, 1]
    p = np.zeros(82, np.uint8)
    p[0], p[1] = 0x00, 0x40                              # d = 2.0
    p[2 + 0], p[2 + 1] = 0xC5, 0x07                      # low index bytes of groups 0, 1
    p[66] = (0x2 << 0) | (0x1 << 2)                      # high bits: group 0 -> 2, group 1 -> 1
    p[34 + 0], p[34 + 1] = 0b10000001, 0b11110000        # signs
    p[74] = 0x3 | (0x9 << 4)                             # ls 3 for groups 0-1, ls 9 for groups 2-3
    y = oracle.decode("iq2_s", grid, p[None])[0]
    assert np.array_equal(y[0:8], 14.0 * np.array([-1, 3, 5, 7, 7, 5, 3, -1]))
    assert np.array_equal(y[8:16], 14.0 * np.array([7, 7, 7, 7, -1, -1, -1, -1]))
    assert np.array_equal(y[16:32], 38.0 * np.ones(16))  # groups 2, 3: entry 0, ls 9, no signs
    assert np.array_equal(y[32:256], 2.0 * np.ones(224))


def test_signs_are_the_inputs(grids):
    w, imp = _case(6, 768, 201)
    p, f = _enc(grids, w, importance=imp)
    assert f == 0
    x = w.float().numpy().reshape(6, 3, 32, 8)
    want = ((x < 0).astype(np.int64) << np.arange(8)).sum(-1)
    got = np.stack([[iq2s_fields(p[r, b])[3] for b in range(3)] for r in range(6)])
    assert np.array_equal(got, want)
    assert ((np.array([bin(v).count("1") for v in want.ravel()]) % 2) == 1).any()  # odd masks exist


@pytest.mark.parametrize("weighted", [False, True])
def test_search_reaches_bruteforce_minimum(grids, weighted):
    w, imp = _case(3, 768, 211)
    if not weighted:
        imp = None
    p, f = _enc(grids, w, importance=imp)
    assert f == 0
    x = w.double().numpy().reshape(3, 3, 256)
    wi = (imp.double().numpy() if imp is not None else np.ones(768)).reshape(3, 256)
    for r in range(3):
        for b in range(3):
            d, ls, idx, s8 = iq2s_fields(p[r, b])
            assert d > 0
            signs = signs_of_mask(s8)
            xb, wb = x[r, b], wi[b]
            for k in range(16):
                objs = [iq2xs_group_objectives(xb[16 * k + 8 * i:16 * k + 8 * i + 8], wb[16 * k + 8 * i:16 * k + 8 * i + 8],
                                               signs[2 * k + i], grids["iq2_s"], d) for i in range(2)]
                per_ls = objs[0].min(1) + objs[1].min(1)
                scale = float((wb[16 * k:16 * k + 16] * xb[16 * k:16 * k + 16] ** 2).sum())
                got = objs[0][ls[k], idx[2 * k]] + objs[1][ls[k], idx[2 * k + 1]]
                assert got <= per_ls.min() + 2e-5 * scale, (r, b, k)


def test_fields_not_degenerate(grids):
    w, imp = _case(16, 1024, 221)
    p, _ = _enc(grids, w, importance=imp)
    ls = np.concatenate([iq2s_fields(b)[1] for b in p.reshape(-1, 82)])
    idx = np.concatenate([iq2s_fields(b)[2] for b in p.reshape(-1, 82)])
    assert len(np.unique(ls)) >= 6 and (idx >= 768).any() and (idx < 1024).all()


def test_lowest_entry_and_ls_win_ties(grids):
    """Columns 0..15 with zero importance: every (ls, entry) scores 0 there -> entry 0, ls 0."""
    w, imp = _case(8, 512, 231)
    imp = imp.clone()
    imp[0:16] = 0.0
    p, f = _enc(grids, w, importance=imp)
    assert f == 0
    for r in range(8):
        _, ls, idx, _ = iq2s_fields(p[r, 0])
        assert ls[0] == 0 and idx[0] == 0 and idx[1] == 0


@pytest.mark.parametrize("c", [2.0, 0.25])
def test_uniform_importance_reproduces_unweighted(grids, c):
    w, _ = _case(6, 512, 241)
    p0, _ = _enc(grids, w)
    p1, _ = _enc(grids, w, importance=torch.full((512,), c))
    np.testing.assert_array_equal(p0, p1)


def test_every_choice_and_fixed_choices(grids):
    w, imp = _case(4, 512, 251)
    every, f = _enc(grids, w, importance=imp, every_choice=True)
    assert f == 0 and every.shape == (16, 4, 2, 82)
    for c in (0, 6, 15):
        fixed, _ = _enc(grids, w, importance=imp, choices=np.full((4, 2, 16), c, np.uint8))
        np.testing.assert_array_equal(every[c], fixed)
    ch = np.random.default_rng(252).integers(0, 16, (4, 2, 16), dtype=np.uint8)
    p, _ = _enc(grids, w, importance=imp, choices=ch)
    for r in range(4):
        for b in range(2):
            _, ls, idx, s8 = iq2s_fields(p[r, b])
            assert (ls == ch[r, b]).all()
            for k in range(16):
                _, _, i2, _ = iq2s_fields(every[ch[r, b, k], r, b])
                assert (idx[2 * k:2 * k + 2] == i2[2 * k:2 * k + 2]).all()


def test_zero_nonfinite_and_range_policy(grids):
    w, imp = _case(3, 1024, 261)
    w[0, 0:256] = 0.0
    w[1, 300] = float("nan")
    w[2, 600] = 3.0e38
    p, f = _enc(grids, w, importance=imp)
    assert not p[0, 0].any() and not p[1, 1].any() and not p[2, 2].any()
    assert f == (1 | 4)
    bad = np.zeros((3, 4, 16), np.uint8)
    bad[2, 3, 0] = 16
    q, f = _enc(grids, w, importance=imp, choices=bad)
    assert f & 8 and not q[2, 3].any()


def test_static_scales_round_trip(grids):
    w, imp = _case(8, 1024, 271)
    p, _ = _enc(grids, w, importance=imp)
    d = np.ascontiguousarray(p[..., 0:2]).view(np.uint16)[..., 0].view(np.float16).astype(np.float64)
    d2 = np.exp2(np.round(np.log2(d))).astype(np.float16)
    pin, _ = _enc(grids, w, importance=imp, scales=d2)
    xhat = oracle.decode("iq2_s", grids["iq2_s"], pin)
    xb = torch.from_numpy(xhat).reshape(8, 1024).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(xhat).reshape(8, 1024))
    q, f = _enc(grids, xb, importance=imp, scales=d2)
    assert f == 0
    np.testing.assert_array_equal(q, pin)
