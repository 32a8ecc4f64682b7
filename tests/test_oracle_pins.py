"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only, no GPU).

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a wrong sign, a
transposed field, a wrong tie-break) fails at least one of them:

* number formats against numpy / torch library conversions;
* the pages' hand-verified IQ1_S example and a hand-built IQ2_XS block (tests/golden);
* the IQ1_S d formula evaluated with numpy's own IEEE fp32/fp16 arithmetic;
* brute force: the oracle's picks reach the fp64 minimum of the direct residual objective;
* invariants named on the pages (non-degenerate fields, d > 0, parity, uniform importance);
* the choice search replayed decision by decision with the direct fp64 block objective.
"""

from __future__ import annotations

import os

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import (block_objective, iq1m_fields, iq1s_fields, iq1s_group_objectives, iq2s_fields, iq2xs_fields,
                       iq2xs_group_objectives, iq2xs_signs, replay_choice_search)
from ggml_iq_codebook_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _case(rows, cols, seed, std=0.02, outlier_frac=0.05, weighted=True):
    w = synth.normal_bf16((rows, cols), std, seed)
    if outlier_frac:
        w = synth.with_outlier_columns(w, synth.outlier_columns(cols, outlier_frac, seed + 1))
    imp = synth.lognormal((cols,), seed + 2) if weighted else None
    return w, imp


def _read_golden(name):
    rec = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        rec.setdefault(key, []).append(vals)
    return rec


# ------------------------------------------------------------------------------ number formats

def test_f32_to_f16_matches_numpy():
    rng = np.random.default_rng(11)
    # exponents around the fp16 range, random mantissas, plus ties and edges
    e = rng.integers(96, 146, size=20000).astype(np.uint32)
    m = rng.integers(0, 1 << 23, size=20000).astype(np.uint32)
    sgn = rng.integers(0, 2, size=20000).astype(np.uint32)
    bits = (sgn << 31) | (e << 23) | m
    vals = list(bits.view(np.float32))
    vals += [0.0, -0.0, 65504.0, 65519.99, 65520.0, 65536.0, 2.0**-14, 2.0**-24, 2.0**-25,
             3 * 2.0**-26, 2.0**-25 * 1.0000001, 1e30, -1e30, 1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11]
    for v in vals:
        v32 = np.float32(v)
        want = int(np.array([v32]).astype(np.float16).view(np.uint16)[0])
        assert oracle.f32_to_f16_bits(float(v32)) == want, v


def test_f16_to_f32_matches_numpy():
    allh = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = allh.view(np.float16).astype(np.float32)
    for h in range(0, 65536, 7):
        if np.isnan(ref[h]):
            continue
        assert oracle.f16_bits_to_f32(h) == ref[h] or (ref[h] == 0 and oracle.f16_bits_to_f32(h) == 0)
        assert np.signbit(oracle.f16_bits_to_f32(h)) == np.signbit(ref[h])


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2**32 - 1, size=200000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16_bits(x), ref)


# ------------------------------------------------------------------------------ layouts (golden)

def test_iq1s_decode_worked_example(grids):
    """d = 2.0, ls = 3 -> scale 14.0, bit 15 -> delta = -0.125, qh = 48712 (PR #2450 review)."""
    g = _read_golden("iq1s_worked_example.txt")
    d_bits = int(g["d_fp16_hex"][0][0], 16)
    qh = int(g["qh"][0][0])
    scale = float(g["scale"][0][0])
    delta = float(g["delta"][0][0])
    high = [int(v) for v in g["high_bits"][0]]
    low = [int(v) for v in g["low"][0]]
    p = np.zeros(50, np.uint8)
    p[0], p[1] = d_bits & 0xFF, d_bits >> 8
    p[2:34] = low
    for k in range(8):
        p[34 + 2 * k], p[35 + 2 * k] = qh & 0xFF, qh >> 8
    y = oracle.decode("iq1_s", grids["iq1_s"], p)
    for grp in range(32):
        idx = low[grp] | (high[grp % 4] << 8)
        want = scale * (grids["iq1_s"][idx].astype(np.float64) + delta)
        assert np.array_equal(y[8 * grp:8 * grp + 8].astype(np.float64), want), grp


def test_iq2xs_decode_hand_built_block(grids):
    g = _read_golden("iq2xs_hand_block.txt")
    d_bits = int(g["d_fp16_hex"][0][0], 16)
    d = float(np.array([d_bits], np.uint16).view(np.float16)[0])
    codes = {int(r[0]): (int(r[1]), int(r[2], 2)) for r in g["code"]}
    for grp in range(32):
        codes.setdefault(grp, ((17 * grp) % 512, grp % 128))
    ls = [int(v) for v in g["ls"][0]]
    p = np.zeros(74, np.uint8)
    p[0], p[1] = d_bits & 0xFF, d_bits >> 8
    for grp, (idx, s7) in codes.items():
        c = idx | (s7 << 9)
        p[2 + 2 * grp], p[3 + 2 * grp] = c & 0xFF, c >> 8
    for i in range(8):
        p[66 + i] = ls[2 * i] | (ls[2 * i + 1] << 4)
    y = oracle.decode("iq2_xs", grids["iq2_xs"], p)
    for grp in range(32):
        idx, s7 = codes[grp]
        bits = [(s7 >> j) & 1 for j in range(7)]
        bits.append(sum(bits) & 1)  # even parity over all 8 signs
        sign = np.array([-1.0 if b else 1.0 for b in bits])
        want = d * (2 * ls[grp // 2] + 1) * grids["iq2_xs"][idx].astype(np.float64) * sign
        assert np.array_equal(y[8 * grp:8 * grp + 8].astype(np.float64), want), grp


# ------------------------------------------------------------------------------ scale d

@pytest.mark.parametrize("fmt,qmax", [("iq1_s", 16.875), ("iq2_xs", 217.0)])
def test_d_formula_numpy_ieee(grids, anchors, fmt, qmax):
    """d = fp16(fp32(amax / qmax) * anchor) with numpy's IEEE fp32 ops and fp16 cast."""
    w, imp = _case(5, 1024, 21)
    p, flags = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    assert flags == 0
    x = w.float().numpy().reshape(5, 4, 256)
    amax = np.abs(x).max(-1).astype(np.float32)
    t = (amax / np.float32(qmax)).astype(np.float32) * np.float32(anchors[fmt])
    want = t.astype(np.float32).astype(np.float16).view(np.uint16)
    got = p[..., 0].astype(np.uint16) | (p[..., 1].astype(np.uint16) << 8)
    assert np.array_equal(got, want)


# ------------------------------------------------------------------------------ brute force

def _iq1s_check_block(x, w, grid, p, tol_rel=2e-5):
    d, ls, neg, idx = iq1s_fields(p)
    assert d > 0
    chosen = ls + 8 * neg
    for k in range(8):
        objs = [iq1s_group_objectives(x[32 * k + 8 * i:32 * k + 8 * i + 8],
                                      w[32 * k + 8 * i:32 * k + 8 * i + 8], grid, d) for i in range(4)]
        per_c = sum(o.min(axis=1) for o in objs)  # [16]
        scale = float((w[32 * k:32 * k + 32] * x[32 * k:32 * k + 32] ** 2).sum()) + 1e-300
        got = sum(objs[i][chosen[k], idx[4 * k + i]] for i in range(4))
        assert got <= per_c.min() + tol_rel * scale, (k, got, per_c.min())
        for i in range(4):
            assert objs[i][chosen[k], idx[4 * k + i]] <= objs[i][chosen[k]].min() + tol_rel * scale


@pytest.mark.parametrize("weighted", [False, True])
def test_iq1s_search_reaches_bruteforce_minimum(grids, anchors, weighted):
    w, imp = _case(3, 768, 31, weighted=weighted)
    p, flags = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], w, importance=imp)
    assert flags == 0
    x = w.double().numpy().reshape(3, 3, 256)
    wi = (imp.double().numpy() if imp is not None else np.ones(768)).reshape(3, 256)
    for r in range(3):
        for b in range(3):
            _iq1s_check_block(x[r, b], wi[b], grids["iq1_s"], p[r, b])


@pytest.mark.parametrize("weighted", [False, True])
def test_iq2xs_search_reaches_bruteforce_minimum(grids, anchors, weighted):
    w, imp = _case(4, 768, 41, std=0.015, weighted=weighted)
    p, flags = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, importance=imp)
    assert flags == 0
    x = w.double().numpy().reshape(4, 3, 256)
    wi = (imp.double().numpy() if imp is not None else np.ones(768)).reshape(3, 256)
    for r in range(4):
        for b in range(3):
            d, ls, idx, s7 = iq2xs_fields(p[r, b])
            signs = iq2xs_signs(s7)  # [32, 8]
            xb, wb = x[r, b], wi[b]
            for grp in range(32):
                xs, ws = xb[8 * grp:8 * grp + 8], wb[8 * grp:8 * grp + 8]
                neg = xs < 0
                flips = np.nonzero((signs[grp] < 0) != neg)[0]
                if neg.sum() % 2 == 0:
                    assert len(flips) == 0
                else:  # exactly one flip, on the weakest element by w x^2
                    assert len(flips) == 1
                    t = ws * xs ** 2
                    assert t[flips[0]] <= t.min() * (1 + 1e-6)
            for k in range(16):
                objs = [iq2xs_group_objectives(xb[16 * k + 8 * i:16 * k + 8 * i + 8],
                                               wb[16 * k + 8 * i:16 * k + 8 * i + 8],
                                               signs[2 * k + i], grids["iq2_xs"], d) for i in range(2)]
                per_ls = objs[0].min(1) + objs[1].min(1)
                scale = float((wb[16 * k:16 * k + 16] * xb[16 * k:16 * k + 16] ** 2).sum())
                got = objs[0][ls[k], idx[2 * k]] + objs[1][ls[k], idx[2 * k + 1]]
                assert got <= per_ls.min() + 2e-5 * scale, (r, b, k)


# ------------------------------------------------------------------------------ invariants

def test_iq1s_fields_not_degenerate(grids, anchors):
    """PR #2450 review: ls and delta take several values, d > 0, and the index fields are really
    used: their high bits (qh bits 0..11) take several values, and every group's decoded entry
    has the sign pattern the group's weights ask for more often than chance (an index read from
    the wrong bits addresses an unrelated grid row)."""
    wl = synth.workload_iq1s_64x256()
    p, flags = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], wl["w"])
    assert flags == 0
    x = wl["w"].float().numpy().reshape(-1, 256)
    f = [iq1s_fields(b) for b in p.reshape(-1, 50)]
    assert all(fi[0] > 0 for fi in f)
    assert len(np.unique(np.concatenate([fi[3] >> 8 for fi in f]))) > 4
    assert len(np.unique(np.concatenate([fi[1] for fi in f]))) > 1
    assert len(np.unique(np.concatenate([fi[2] for fi in f]))) == 2
    # the entry of a group tracks the signs of its largest weights: count, over all groups, the
    # elements whose grid value has the weight's sign among the 2 largest |x| of the group
    agree = total = 0
    for blk, fi in zip(x, f):
        q = grids["iq1_s"][fi[3]].astype(np.int64)  # [32, 8]
        xg = blk.reshape(32, 8)
        top = np.argsort(-np.abs(xg), axis=1)[:, :2]
        for g in range(32):
            for j in top[g]:
                total += 1
                agree += int(np.sign(q[g, j]) == np.sign(xg[g, j]))
    assert agree > 0.8 * total, (agree, total)


def test_iq2xs_fields_not_degenerate(grids, anchors):
    """PR #2450 review: the decoded signs are the input's signs up to the one weakest flip an odd
    count needs, the scale nibbles are not all equal, the 9-bit indices use their top bit, and
    d > 0."""
    w, imp = _case(16, 256, 51, std=0.015)
    p, flags = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, importance=imp)
    assert flags == 0
    x = w.float().numpy().reshape(-1, 256)
    tops = set()
    for blk, xb in zip(p.reshape(-1, 74), x):
        d, ls, idx, s7 = iq2xs_fields(blk)
        assert d > 0
        assert len(np.unique(ls)) > 1
        tops |= set((idx >> 8).tolist())
        dec_neg = iq2xs_signs(s7) < 0           # [32, 8]
        in_neg = xb.reshape(32, 8) < 0
        diff = (dec_neg != in_neg).sum(-1)      # elements whose sign the encoder changed
        assert np.array_equal(diff, in_neg.sum(-1) % 2), (diff, in_neg.sum(-1))
    assert tops == {0, 1}


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("c", [1.0, 2.0, 0.25])
def test_uniform_importance_reproduces_unweighted(grids, anchors, fmt, c):
    """PR #2723: uniform importance gives the unweighted payload exactly (power-of-two c)."""
    w, _ = _case(6, 512, 61, weighted=False)
    p0, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w)
    p1, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=np.full(512, c, np.float32))
    assert np.array_equal(p0, p1)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_decode_is_exact(grids, anchors, fmt):
    """Every decoded value is the exact product d * (2 ls + 1) * (grid value [+ delta])."""
    w, imp = _case(4, 512, 71)
    p, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    y = oracle.decode(fmt, grids[fmt], p).astype(np.float64)
    for r in range(4):
        for b in range(2):
            if fmt == "iq1_s":
                d, ls, neg, idx = iq1s_fields(p[r, b])
                for grp in range(32):
                    k = grp // 4
                    want = d * (2 * ls[k] + 1) * (grids[fmt][idx[grp]] + (-0.125 if neg[k] else 0.125))
                    assert np.array_equal(y[r, b, 8 * grp:8 * grp + 8], want)
            else:
                d, ls, idx, s7 = iq2xs_fields(p[r, b])
                sg = iq2xs_signs(s7)
                for grp in range(32):
                    want = d * (2 * ls[grp // 2] + 1) * grids[fmt][idx[grp]] * sg[grp]
                    assert np.array_equal(y[r, b, 8 * grp:8 * grp + 8], want)


# ------------------------------------------------------------------------------ fixed choices

@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_fixed_choices(grids, anchors, fmt):
    """PR #3157: under fixed choices each group's fields equal those of the encode that forces its
    choice on every group."""
    G = oracle.CHOICE_GROUPS[fmt]
    w, imp = _case(3, 512, 81)
    p, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    own = _choices_of(fmt, p)
    p_own, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, choices=own)
    assert np.array_equal(p_own, p)
    every, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    rng = np.random.default_rng(5)
    ch = rng.integers(0, 16, size=(3, 2, G)).astype(np.uint8)
    pf, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, choices=ch)
    for r in range(3):
        for b in range(2):
            for k in range(G):
                ref = every[ch[r, b, k], r, b]
                _assert_group_fields_equal(fmt, pf[r, b], ref, k)
    # and the forced entries are the fp64 best under the forced choice (IQ1_S)
    if fmt == "iq1_s":
        x = w.double().numpy().reshape(3, 2, 256)
        wi = imp.double().numpy().reshape(2, 256)
        for r in range(3):
            for b in range(2):
                d, ls, neg, idx = iq1s_fields(pf[r, b])
                assert np.array_equal(ls + 8 * neg, ch[r, b])
                for grp in range(32):
                    o = iq1s_group_objectives(x[r, b, 8 * grp:8 * grp + 8], wi[b, 8 * grp:8 * grp + 8],
                                              grids[fmt], d)[ch[r, b, grp // 4]]
                    assert o[idx[grp]] <= o.min() + 2e-5 * (np.abs(o).max())


def _choices_of(fmt, p):
    G = oracle.CHOICE_GROUPS[fmt]
    out = np.zeros(p.shape[:-1] + (G,), np.uint8)
    for i in np.ndindex(p.shape[:-1]):
        if fmt == "iq1_s":
            _, ls, neg, _ = iq1s_fields(p[i])
            out[i] = ls + 8 * neg
        elif fmt == "iq2_s":
            out[i] = iq2s_fields(p[i])[1]
        elif fmt == "iq1_m":
            out[i] = iq1m_fields(p[i])[1]
        else:
            out[i] = iq2xs_fields(p[i])[1]
    return out


def _assert_group_fields_equal(fmt, a, b, k):
    assert a[0] == b[0] and a[1] == b[1]
    assert np.array_equal(a[2 + 4 * k:6 + 4 * k], b[2 + 4 * k:6 + 4 * k])
    if fmt == "iq1_s":
        assert np.array_equal(a[34 + 2 * k:36 + 2 * k], b[34 + 2 * k:36 + 2 * k])
    else:
        sh = 4 * (k & 1)
        assert (a[66 + k // 2] >> sh) & 15 == (b[66 + k // 2] >> sh) & 15


# ------------------------------------------------------------------------------ zero / errors

@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_zero_nonfinite_and_range_policy(grids, anchors, fmt):
    B = oracle.BLOCK_BYTES[fmt]
    w, imp = _case(6, 256, 91, weighted=True)
    w = w.clone()
    w[1] = 0.0                        # all-zero block: all-zero payload, no flag
    w[2] = 1e-7                       # d underflows fp16: zero payload, no flag
    w[3, 17] = float("nan")           # non-finite weight
    w[4, 5] = float("inf")
    w[5, 0] = 3e9                     # d overflows fp16
    ref, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w[:1], importance=imp)
    p, flags = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    assert flags == oracle.FLAG_NONFINITE | oracle.FLAG_RANGE
    assert np.array_equal(p[0], ref[0])
    for r in range(1, 6):
        assert not p[r].any(), r
    bad = imp.clone()
    bad[3] = -1.0
    p, flags = oracle.encode(fmt, grids[fmt], anchors[fmt], w[:1], importance=bad)
    assert flags == oracle.FLAG_IMPORTANCE and not p.any()
    ch = np.full((1, 1, oracle.CHOICE_GROUPS[fmt]), 16, np.uint8)
    p, flags = oracle.encode(fmt, grids[fmt], anchors[fmt], w[:1], importance=imp, choices=ch)
    assert flags == oracle.FLAG_CHOICE and p.shape == (1, 1, B) and not p.any()


# ------------------------------------------------------------------------------ choice search

def _choice_case(fmt, grids, anchors, rows, nblk, seed, offdiag):
    w = synth.normal_bf16((rows, nblk * 256), 0.02, seed)
    hess = torch.stack([synth.block_hessian(seed + 10 + b, offdiag_std=offdiag) for b in range(nblk)]).numpy()
    imp = oracle.sqrt_diag(hess)
    cand, flags = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    assert flags == 0
    return w, hess, cand


def _deltas(fmt, grids, w, cand, r, b):
    x = w.double().numpy()[r, 256 * b:256 * b + 256]
    xh = oracle.decode(fmt, grids[fmt], cand[:, r, b]).astype(np.float64)  # [16, 256]
    return x[None] - xh


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
@pytest.mark.parametrize("offdiag", [0.02, 0.3])
def test_choice_search_decisions_replay_in_fp64(grids, anchors, fmt, offdiag):
    """PR #3158: step 2 and both sweeps, checked decision by decision on the direct objective."""
    rows, nblk = (6, 2) if fmt == "iq2_xs" else (3, 2)
    w, hess, cand = _choice_case(fmt, grids, anchors, rows, nblk, 101, offdiag)
    picks, payload, trace = oracle.choice_search(fmt, grids[fmt], w, hess, cand, trace=True)
    G = oracle.CHOICE_GROUPS[fmt]
    total_switches = 0
    for r in range(rows):
        for b in range(nblk):
            viol, sw, objs = replay_choice_search(_deltas(fmt, grids, w, cand, r, b), hess[b], G,
                                                  trace[r, b], rel_tol=3e-5)
            assert not viol, viol
            assert objs[2] <= objs[1] * (1 + 1e-6) and objs[1] <= objs[0] * (1 + 1e-6)
            total_switches += sw
            assert np.array_equal(picks[r, b], trace[r, b, 2])
    if offdiag > 0.1:
        assert total_switches > 0  # the sweeps do something on correlated inputs


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
def test_choice_search_block_diagonal_hessian_makes_sweeps_noops(grids, anchors, fmt):
    G = oracle.CHOICE_GROUPS[fmt]
    W = 256 // G
    w, hess, cand = _choice_case(fmt, grids, anchors, 3, 1, 111, 0.3)
    mask = np.kron(np.eye(G), np.ones((W, W))).astype(np.float32)
    hb = hess * mask[None]
    picks, payload, trace = oracle.choice_search(fmt, grids[fmt], w, hb, cand, trace=True)
    assert np.array_equal(trace[..., 0, :], trace[..., 1, :])
    assert np.array_equal(trace[..., 0, :], trace[..., 2, :])


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
def test_choice_search_identity_hessian_keeps_encoder_choices(grids, anchors, fmt):
    """PR #3158: under H = I (with unit importance) the search keeps the encoder's own choices."""
    rows = 2 if fmt == "iq1_s" else 4
    w = synth.normal_bf16((rows, 256), 0.02, 121)
    hess = np.eye(256, dtype=np.float32)[None]
    cand, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, every_choice=True)
    own, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w)
    picks, payload = oracle.choice_search(fmt, grids[fmt], w, hess, cand)
    want = _choices_of(fmt, own)
    G = oracle.CHOICE_GROUPS[fmt]
    W = 256 // G
    for r in range(rows):
        dl = _deltas(fmt, grids, w, cand, r, 0)
        for g in range(G):
            if picks[r, 0, g] != want[r, 0, g]:
                sl = slice(g * W, g * W + W)
                a = float((dl[picks[r, 0, g], sl] ** 2).sum())
                bb = float((dl[want[r, 0, g], sl] ** 2).sum())
                assert abs(a - bb) <= 1e-5 * max(a, bb), (r, g)  # only an fp near-tie may differ


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
def test_choice_search_payload_is_the_encode_under_picks(grids, anchors, fmt):
    """PR #3157 + #3158: the final payload equals quantize(..., choices=picks)."""
    w, hess, cand = _choice_case(fmt, grids, anchors, 3, 2, 131, 0.3)
    picks, payload = oracle.choice_search(fmt, grids[fmt], w, hess, cand)
    imp = oracle.sqrt_diag(hess)
    enc, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, choices=picks)
    assert np.array_equal(payload, enc)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s"])
def test_choice_search_experts_use_their_own_hessians(grids, anchors, fmt):
    """A stack of experts in one call equals one call per expert with that expert's H, and each
    expert's decisions replay against its own H (the regime PR #3218 targets: many small
    expert weights)."""
    nexp, rows, nblk = 3, 3, 2
    w = synth.normal_bf16((nexp, rows, nblk * 256), 0.02, 141)
    hess = np.stack([np.stack([synth.block_hessian(150 + 10 * e + b, offdiag_std=0.3).numpy() for b in range(nblk)])
                     for e in range(nexp)])                           # [E, nblk, 256, 256]
    imp = oracle.sqrt_diag(hess).reshape(nexp, nblk * 256)
    cand = np.stack([oracle.encode(fmt, grids[fmt], anchors[fmt], w[e], importance=imp[e], every_choice=True)[0]
                     for e in range(nexp)], axis=1)                   # [16, E, rows, nblk, B]
    picks, payload, trace = oracle.choice_search(fmt, grids[fmt], w, hess, cand, trace=True)
    assert picks.shape[:3] == (nexp, rows, nblk)
    G = oracle.CHOICE_GROUPS[fmt]
    for e in range(nexp):
        pe, ye = oracle.choice_search(fmt, grids[fmt], w[e], hess[e], cand[:, e])
        assert np.array_equal(picks[e], pe) and np.array_equal(payload[e], ye)
        for r in range(rows):
            for b in range(nblk):
                x = w[e].double().numpy()[r, 256 * b:256 * b + 256]
                dl = x[None] - oracle.decode(fmt, grids[fmt], cand[:, e, r, b]).astype(np.float64)
                viol, _, _ = replay_choice_search(dl, hess[e, b], G, trace[e, r, b], rel_tol=3e-5)
                assert not viol, viol
    other, _ = oracle.choice_search(fmt, grids[fmt], w, hess[[1, 2, 0]], cand)
    assert not np.array_equal(other, picks)           # the Hessians do reach the decisions


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m"])
def test_choice_search_objective_is_the_final_quadratic_form(grids, anchors, fmt):
    """The reported objective, sum_i Delta_i grad_i with the incrementally updated gradient,
    equals Delta^T H Delta of the final payload recomputed in fp64 from scratch."""
    w, hess, cand = _choice_case(fmt, grids, anchors, 4, 2, 151, 0.3)
    picks, payload, obj = oracle.choice_search(fmt, grids[fmt], w, hess, cand, objective=True)
    xh = oracle.decode(fmt, grids[fmt], payload).astype(np.float64)           # [rows, nblk, 256]
    x = w.double().numpy().reshape(4, 2, 256)
    for r in range(4):
        for b in range(2):
            dl = x[r, b] - xh[r, b]
            H = hess[b].astype(np.float64)
            scale = np.abs(dl) @ np.abs(H) @ np.abs(dl)
            assert abs(float(obj[r, b]) - dl @ H @ dl) <= 1e-5 * scale, (r, b)


def test_sqrt_diag_matches_numpy():
    h = torch.stack([synth.block_hessian(7), synth.block_hessian(8)]).numpy()
    want = np.sqrt(np.stack([np.diag(h[0]), np.diag(h[1])]).astype(np.float32)).reshape(-1)
    assert np.array_equal(oracle.sqrt_diag(h), want)


def test_hessian_recipe_is_symmetric_and_well_conditioned():
    h = synth.block_hessian(5000).numpy().astype(np.float64)
    assert np.array_equal(h, h.T)
    ev = np.linalg.eigvalsh(h)
    assert ev.min() > 0 and ev.max() / ev.min() < 100


def test_block_objective_is_quadratic_form():
    rng = np.random.default_rng(3)
    a = rng.normal(size=(256, 256))
    h = a @ a.T
    v = rng.normal(size=256)
    assert np.isclose(block_objective(v, h), float(np.einsum("i,ij,j->", v, h, v)))


# ------------------------------------------------------------------------------ tie-breaks

def test_iq1s_lowest_index_wins_on_equal_error(grids, anchors):
    """PR #2450 review: on equal error the lower index is taken. With zero importance on two columns of
    each group, entries that differ only there tie exactly (also in fp64); the lowest must win.
    A sub-block with zero importance everywhere ties on every (entry, choice): choice 0, entry 0."""
    w, _ = _case(2, 256, 141, weighted=False)
    imp = np.ones(256, np.float32)
    imp[6::8] = 0.0
    imp[7::8] = 0.0
    imp[64:96] = 0.0
    p, flags = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], w, importance=imp)
    assert flags == 0
    x = w.double().numpy()
    grid = grids["iq1_s"]
    tied = 0
    for r in range(2):
        d, ls, neg, idx = iq1s_fields(p[r, 0])
        assert ls[2] == 0 and neg[2] == 0 and not idx[8:12].any()
        for grp in range(32):
            if 8 <= grp < 12:
                continue
            c = ls[grp // 4] + 8 * neg[grp // 4]
            o = iq1s_group_objectives(x[r, 8 * grp:8 * grp + 8], imp[8 * grp:8 * grp + 8], grid, d)[c]
            ties = np.nonzero(o == o[idx[grp]])[0]
            assert idx[grp] == ties.min(), grp
            tied += len(ties) >= 2
    assert tied >= 8


def test_iq2xs_lowest_index_wins_on_equal_error(grids, anchors):
    w, _ = _case(2, 256, 151, std=0.015, weighted=False)
    imp = np.ones(256, np.float32)
    for j in (1, 3, 4, 6):  # the 512-entry grid is sparse in {1,3,5,7}^8: tie four columns
        imp[j::8] = 0.0
    imp[32:48] = 0.0
    p, flags = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], w, importance=imp)
    assert flags == 0
    x = w.double().numpy()
    tied = 0
    for r in range(2):
        d, ls, idx, s7 = iq2xs_fields(p[r, 0])
        assert ls[2] == 0 and not idx[4:6].any()
        sg = iq2xs_signs(s7)
        for grp in range(32):
            if grp in (4, 5):
                continue
            o = iq2xs_group_objectives(x[r, 8 * grp:8 * grp + 8], imp[8 * grp:8 * grp + 8], sg[grp],
                                       grids["iq2_xs"], d)[ls[grp // 2]]
            ties = np.nonzero(o == o[idx[grp]])[0]
            assert idx[grp] == ties.min(), grp
            tied += len(ties) >= 2
    assert tied >= 8


# ------------------------------------------------------------------------------ joint enumeration

def test_iq1s_joint_enumeration_on_a_reduced_grid(anchors):
    """A 2048-entry grid holding only 16 distinct rows (each repeated) lets fp64 enumerate every
    (choice, entry of each of the 4 groups) of a whole 32-weight sub-block jointly: 16 x 16^4
    candidates. The oracle's separable search must reach that joint minimum."""
    rng = np.random.default_rng(161)
    rows16 = np.stack([rng.integers(-1, 2, 8) for _ in range(16)]).astype(np.int8)
    grid = np.tile(rows16, (128, 1))                      # entry q is row q % 16
    w, imp = _case(1, 256, 162)
    p, f = oracle.encode("iq1_s", grid, anchors["iq1_s"], w, importance=imp)
    assert f == 0
    x, wi = w.double().numpy()[0], imp.double().numpy()
    d, ls, neg, idx = iq1s_fields(p[0, 0])
    for k in range(2):                                    # two sub-blocks, enumerated jointly
        xs, ws = x[32 * k:32 * k + 32].reshape(4, 8), wi[32 * k:32 * k + 32].reshape(4, 8)
        best = np.inf
        for c in range(16):
            s = d * (2 * (c & 7) + 1)
            delta = -0.125 if c >= 8 else 0.125
            xhat = s * (rows16.astype(np.float64) + delta)                     # [16, 8]
            e = ((xs[:, None, :] - xhat[None]) ** 2 * ws[:, None, :]).sum(-1)  # [4 groups, 16]
            joint = (e[0][:, None, None, None] + e[1][None, :, None, None]
                     + e[2][None, None, :, None] + e[3][None, None, None, :])  # all 16^4 combinations
            best = min(best, joint.min())
        c = ls[k] + 8 * neg[k]
        s = d * (2 * (c & 7) + 1)
        delta = -0.125 if c >= 8 else 0.125
        got = sum(float(((xs[i] - s * (grid[idx[4 * k + i]] + delta)) ** 2 * ws[i]).sum()) for i in range(4))
        scale = float((ws * xs ** 2).sum())
        assert got <= best + 2e-5 * scale, (k, got, best)
        assert all(idx[4 * k + i] < 16 for i in range(4))  # ties resolve to the first copy of a row


def test_iq2xs_joint_enumeration_on_a_reduced_grid(anchors):
    """512 entries made of 16 distinct magnitude rows: fp64 enumerates every (ls, entry, entry) of
    a 16-weight sub-block jointly (16 x 16^2) under the signs the encoder fixed; the oracle must
    reach that minimum, and repeated rows resolve to their first copy."""
    rng = np.random.default_rng(171)
    rows16 = np.stack([rng.choice([1, 3, 5, 7], 8) for _ in range(16)]).astype(np.int8)
    grid = np.tile(rows16, (32, 1))
    w, imp = _case(1, 256, 172, std=0.015)
    p, f = oracle.encode("iq2_xs", grid, anchors["iq2_xs"], w, importance=imp)
    assert f == 0
    x, wi = w.double().numpy()[0], imp.double().numpy()
    d, ls, idx, s7 = iq2xs_fields(p[0, 0])
    signs = iq2xs_signs(s7)
    for k in range(4):
        xs, ws = x[16 * k:16 * k + 16].reshape(2, 8), wi[16 * k:16 * k + 16].reshape(2, 8)
        best = np.inf
        for l in range(16):
            s = d * (2 * l + 1)
            e = [((xs[i][None] - s * rows16 * signs[2 * k + i][None]) ** 2 * ws[i][None]).sum(-1) for i in range(2)]
            best = min(best, (e[0][:, None] + e[1][None, :]).min())
        s = d * (2 * ls[k] + 1)
        got = sum(float(((xs[i] - s * grid[idx[2 * k + i]] * signs[2 * k + i]) ** 2 * ws[i]).sum()) for i in range(2))
        assert got <= best + 2e-5 * float((ws * xs ** 2).sum()), (k, got, best)
        assert idx[2 * k] < 16 and idx[2 * k + 1] < 16


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m", "g8"])
def test_choice_search_ties_go_to_the_lowest_choice(grids, anchors, fmt):
    """PR #3158's tie rules on exact ties: a candidate duplicated at a higher choice scores and
    gains exactly what its lower copy does, so it is never picked (lowest choice on equal score,
    and a switch needs a strictly negative gain); with every candidate equal nothing moves."""
    efmt = "iq2_xs" if fmt == "g8" else fmt
    w, hess, cand = _choice_case(efmt, grids, anchors, 4, 2, 161, 0.3)
    C = cand.shape[0]
    lo = 8 if fmt == "g8" else 0                      # first candidate the search reads

    def search(cd):
        if fmt == "g8":
            return oracle.choice_search_g8(grids["iq2_xs"], w, hess, cd, trace=True)[1]
        return oracle.choice_search(fmt, grids[fmt], w, hess, cd, trace=True)[2]

    dup = cand.copy()
    pairs = [(lo + 1, C - 1), (lo + 2, lo + 4)]       # (kept copy, higher duplicate)
    for keep, high in pairs:
        dup[high] = dup[keep]
    tr = search(dup)
    for _, high in pairs:
        assert not (tr == high).any(), high
    same = np.broadcast_to(cand[lo:lo + 1], cand.shape).copy()
    tr = search(same)
    assert (tr == lo).all()


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "g8"])
def test_choice_search_findings_policy(grids, anchors, fmt):
    """A non-finite weight taints its own row-block, a non-finite Hessian entry every row-block of
    that Hessian block, a grid value outside the alphabet every block: those get picks 0 (the first
    candidate), the all-zero payload and a NaN objective, with the finding flagged; the other
    row-blocks are exactly what they are without the bad input."""
    base = "iq2_xs" if fmt == "g8" else fmt
    w, hess, cand = _choice_case(base, grids, anchors, 4, 2, 131, 0.3)

    def run(w_, h_, g_):
        if fmt == "g8":
            picks, obj, flags = oracle.choice_search_g8(g_, w_, h_, cand, objective=True, return_flags=True)
            return picks, None, obj, flags
        return oracle.choice_search(fmt, g_, w_, h_, cand, objective=True, return_flags=True)

    picks0, pay0, obj0, f0 = run(w, hess, grids[base])
    assert f0 == 0
    first = 8 if fmt == "g8" else 0
    nan_bits = np.uint32(0x7FC00000)
    wb = w.clone()
    wb[1, 300] = float("nan")                      # row 1, block 1
    hb = hess.copy()
    hb[0, 7, 9] = np.inf                           # block 0 of every row
    picks, pay, obj, f = run(wb, hb, grids[base])
    assert f == oracle.FLAG_NONFINITE
    bad = np.zeros((4, 2), bool)
    bad[:, 0] = True
    bad[1, 1] = True
    assert np.all(picks[bad] == first) and np.all(obj.view(np.uint32)[bad] == nan_bits)
    assert np.array_equal(picks[~bad], picks0[~bad]) and np.array_equal(obj[~bad], obj0[~bad])
    if pay is not None:
        assert not pay[bad].any() and np.array_equal(pay[~bad], pay0[~bad])
    g_bad = grids[base].copy()
    g_bad[3, 2] = 2 if base != "iq1_s" else -2     # outside {1,3,5,7} / {-1,0,1}
    picks, pay, obj, f = run(w, hess, g_bad)
    assert f == oracle.FLAG_GRID
    assert np.all(picks == first) and np.all(obj.view(np.uint32) == nan_bits)
    if pay is not None:
        assert not pay.any()
