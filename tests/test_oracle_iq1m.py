"""Pins of the oracle's IQ1_M encoder and decoder (CPU only, no GPU).

IQ1_M (PR #2513 codec and PR #2595 CUDA encoder commit texts, on the page of PR #2525): the IQ1_S
shifted-grid search, a local scale per two groups, a delta per group, d stored as the top nibbles
of four scale words, and the anchor clamp(0.58 + 0.035 * peak_to_rms, 0.65, 0.95). What fixes it:

* the anchor points PR #2513's test uses: blocks built with peak-to-RMS ratios of 1, 4, 8 and 16
  reach both clamps and two points on the slope, with d computed here in numpy's IEEE fp32/fp16;
* a hand-built block decoded against values written out from the layout reading;
* fp64 brute force: every pick reaches the minimum of the direct residual over (ls, delta, entry);
* the tie order the pages state (lower shift, then lower entry), uniform-importance invariance,
  every-choice == fixed choices, the zero and range policy, and the static-scale round trip.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import iq1m_fields, iq1s_group_objectives
from ggml_iq_codebook_b200 import synth

F32 = np.float32


def _case(rows, cols, seed, std=0.02):
    w = synth.normal_bf16((rows, cols), std, seed)
    w = synth.with_outlier_columns(w, synth.outlier_columns(cols, 0.05, seed + 1))
    return w, synth.lognormal((cols,), seed + 2)


def _enc(grids, w, **kw):
    return oracle.encode("iq1_m", grids["iq1_s"], 0.0, w, **kw)


@pytest.mark.parametrize("ratio,anchor_expected", [(1, 0.65), (4, 0.72), (8, 0.86), (16, 0.95)])
def test_anchor_follows_peak_to_rms(grids, ratio, anchor_expected):
    """The anchor at peak-to-RMS 1, 4, 8 and 16 (PR #2513's test points): both clamps, two slope points."""
    n = 256 // (ratio * ratio)                       # n unit spikes in 256 weights: rms = sqrt(n/256)
    amax = 0.375
    x = np.zeros((1, 256), np.float32)
    pos = np.random.default_rng(ratio).permutation(256)[:n]
    x[0, pos] = amax * np.where(np.arange(n) % 2 == 0, 1.0, -1.0)
    p, f = _enc(grids, torch.from_numpy(x).bfloat16())
    assert f == 0
    a = np.minimum(np.maximum(F32(0.58) + F32(0.035) * F32(ratio), F32(0.65)), F32(0.95))
    assert abs(float(a) - anchor_expected) < 1e-6
    d_expected = np.float16(F32(F32(amax) / F32(16.875)) * a)
    d, _, _, _ = iq1m_fields(p[0, 0])
    assert d == float(d_expected), (d, float(d_expected))


def test_decode_hand_built_block():
    """Fields written by hand from the layout reading; values d (2 ls + 1)(q + delta) by hand."""
    grid = np.zeros((2048, 8), np.int8)
    grid[0x2A5] = [1, -1, 0, 0, 1, 1, -1, 0]
    grid[0x13] = [-1, -1, -1, -1, 1, 1, 1, 1]
    grid[0x700] = [0, 0, 0, 0, 0, 0, 0, 1]
    p = np.zeros(56, np.uint8)
    # d = 2.0 = fp16 0x4000: nibbles 0, 0, 0, 4 in the top of scale words 0..3
    # group 0: entry 0x2A5, delta -1/8; group 1: entry 0x013, delta +1/8; pair 0 (groups 0, 1): ls 3
    # group 5: entry 0x700, delta -1/8; pair 2 (groups 4, 5): ls 6
    p[0], p[1], p[5] = 0xA5, 0x13, 0x00
    p[32] = (0x2 | 0x8) | (0x0 << 4)
    p[34] = 0x0 | ((0x7 | 0x8) << 4)
    word0 = 3 | (6 << 6)                              # ls of pair 0 at shift 0, pair 2 at shift 6
    p[48], p[49] = word0 & 0xFF, word0 >> 8
    p[54], p[55] = 0x00, 0x40                         # word 3 = 0x4000: d's top nibble
    y = oracle.decode("iq1_m", grid, p[None])[0]
    assert np.array_equal(y[0:8], 14.0 * (np.array([1, -1, 0, 0, 1, 1, -1, 0]) - 0.125))
    assert np.array_equal(y[8:16], 14.0 * (np.array([-1, -1, -1, -1, 1, 1, 1, 1]) + 0.125))
    assert np.array_equal(y[40:48], 26.0 * (np.array([0, 0, 0, 0, 0, 0, 0, 1]) - 0.125))
    assert np.array_equal(y[32:40], 26.0 * 0.125 * np.ones(8))       # group 4: entry 0, delta +1/8
    assert np.array_equal(y[16:32], 2.0 * 0.125 * np.ones(16))       # pair 1: ls 0, entry 0


def _check_block(x, w, grid, p, tol=2e-5):
    d, ls, neg, idx = iq1m_fields(p)
    assert d > 0
    for k in range(16):
        objs = [iq1s_group_objectives(x[16 * k + 8 * i:16 * k + 8 * i + 8], w[16 * k + 8 * i:16 * k + 8 * i + 8],
                                      grid, d) for i in range(2)]            # [16 = ls + 8 neg, 2048]
        per_ls = [sum(min(o[l].min(), o[l + 8].min()) for o in objs) for l in range(8)]
        scale = float((w[16 * k:16 * k + 16] * x[16 * k:16 * k + 16] ** 2).sum()) + 1e-300
        got = sum(objs[i][ls[k] + 8 * neg[2 * k + i], idx[2 * k + i]] for i in range(2))
        assert got <= min(per_ls) + tol * scale, (k, got, min(per_ls))
        for i in range(2):
            o = objs[i]
            assert o[ls[k] + 8 * neg[2 * k + i], idx[2 * k + i]] <= min(o[ls[k]].min(), o[ls[k] + 8].min()) + tol * scale


@pytest.mark.parametrize("weighted", [False, True])
def test_search_reaches_bruteforce_minimum(grids, weighted):
    w, imp = _case(3, 768, 121)
    if not weighted:
        imp = None
    p, f = _enc(grids, w, importance=imp)
    assert f == 0
    x = w.double().numpy().reshape(3, 3, 256)
    wi = (imp.double().numpy() if imp is not None else np.ones(768)).reshape(3, 256)
    for r in range(3):
        for b in range(3):
            _check_block(x[r, b], wi[b], grids["iq1_s"], p[r, b])


def test_fields_not_degenerate(grids):
    w, imp = _case(16, 1024, 131)
    p, _ = _enc(grids, w, importance=imp)
    ls, neg = [], []
    for blk in p.reshape(-1, 56):
        d, l, n, idx = iq1m_fields(blk)
        assert d > 0 and (idx < 2048).all()
        ls.append(l)
        neg.append(n)
    ls, neg = np.concatenate(ls), np.concatenate(neg)
    assert len(np.unique(ls)) >= 4 and 0.2 < neg.mean() < 0.8


def test_lower_shift_then_lower_entry_win_ties(grids):
    """A group whose importance is all zero has m = 0 for every (delta, entry): +1/8 and entry 0."""
    w, imp = _case(8, 512, 141)
    imp = imp.clone()
    imp[0:8] = 0.0
    imp[256 + 40:256 + 48] = 0.0
    p, f = _enc(grids, w, importance=imp)
    assert f == 0
    for r in range(8):
        _, _, neg, idx = iq1m_fields(p[r, 0])
        assert neg[0] == 0 and idx[0] == 0
        _, _, neg, idx = iq1m_fields(p[r, 1])
        assert neg[5] == 0 and idx[5] == 0


@pytest.mark.parametrize("c", [2.0, 0.25])
def test_uniform_importance_reproduces_unweighted(grids, c):
    w, _ = _case(6, 512, 151)
    p0, _ = _enc(grids, w)
    p1, _ = _enc(grids, w, importance=torch.full((512,), c))
    np.testing.assert_array_equal(p0, p1)


def test_every_choice_matches_fixed_choices(grids):
    w, imp = _case(4, 512, 161)
    every, f = _enc(grids, w, importance=imp, every_choice=True)
    assert f == 0 and every.shape == (8, 4, 2, 56)
    for c in range(8):
        fixed, _ = _enc(grids, w, importance=imp, choices=np.full((4, 2, 16), c, np.uint8))
        np.testing.assert_array_equal(every[c], fixed)
        for blk in fixed.reshape(-1, 56):
            assert (iq1m_fields(blk)[1] == c).all()


def test_fixed_choices_per_group(grids):
    w, imp = _case(5, 768, 171)
    ch = np.random.default_rng(172).integers(0, 8, (5, 3, 16), dtype=np.uint8)
    p, f = _enc(grids, w, importance=imp, choices=ch)
    assert f == 0
    every, _ = _enc(grids, w, importance=imp, every_choice=True)
    for r in range(5):
        for b in range(3):
            _, ls, neg, idx = iq1m_fields(p[r, b])
            assert (ls == ch[r, b]).all()
            for k in range(16):
                _, _, n2, i2 = iq1m_fields(every[ch[r, b, k], r, b])
                assert (neg[2 * k:2 * k + 2] == n2[2 * k:2 * k + 2]).all()
                assert (idx[2 * k:2 * k + 2] == i2[2 * k:2 * k + 2]).all()
    bad = ch.copy()
    bad[1, 2, 7] = 8
    q, f = _enc(grids, w, importance=imp, choices=bad)
    assert f == 8 and not q[1, 2].any() and (q[0] == p[0]).all()


def test_zero_nonfinite_and_range_policy(grids):
    w, imp = _case(3, 1024, 181)
    w[0, 0:256] = 0.0
    w[1, 300] = float("inf")
    w[2, 600] = 6.0e4                              # amax / 16.875 * 0.95 overflows fp16 past 65504
    w[2, 512:768] = 0.0
    w[2, 600] = 3.0e38
    p, f = _enc(grids, w, importance=imp)
    assert not p[0, 0].any() and not p[1, 1].any() and not p[2, 2].any()
    assert f == (1 | 4)
    assert p[0, 1].any() and p[1, 0].any()


def test_static_scales_round_trip(grids):
    w, imp = _case(8, 1024, 191)
    p, _ = _enc(grids, w, importance=imp)
    d = np.array([[iq1m_fields(b)[0] for b in row] for row in p], np.float64)
    d2 = np.exp2(np.round(np.log2(d))).astype(np.float16)
    pin, _ = _enc(grids, w, importance=imp, scales=d2)
    xhat = oracle.decode("iq1_m", grids["iq1_s"], pin)
    xb = torch.from_numpy(xhat).reshape(8, 1024).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(xhat).reshape(8, 1024))
    q, f = _enc(grids, xb, importance=imp, scales=d2)
    assert f == 0
    np.testing.assert_array_equal(q, pin)
