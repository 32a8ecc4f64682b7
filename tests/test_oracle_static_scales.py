"""Pins of the oracle's static-scale encode (CPU only, no GPU).

PR #3197 ("... QAD starts from GPTQ's and imatrix's codes", its "Static scales" item): a pinned
weight is re-encoded under the block scales d it was first packed with, and a weight and its
decoding both re-encode to the pinned codes. What fixes the oracle here:

* given d equal to the predicted one reproduces the predicted-d payload byte for byte;
* decoding a payload whose d is a power of two gives values that bf16 holds exactly (|(2 ls + 1)
  (8 q + 8 delta)| <= 135 and (2 ls + 1) g <= 105 need at most 8 significant bits), so the
  re-encode under the same d must reach zero error: it decodes to the same values, and is
  byte-identical since no other code decodes to the same values;
* under a d unrelated to amax, the picks still reach the fp64 brute-force minimum;
* the policy for refused scales (negative, infinite, NaN), +-0 and all-zero blocks.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import iq1s_fields, iq1s_group_objectives, iq2xs_fields, iq2xs_group_objectives, iq2xs_signs
from ggml_iq_codebook_b200 import synth

B = {"iq1_s": 50, "iq2_xs": 74}
FLAG_RANGE = 4


def _case(rows, cols, seed, std=0.02):
    w = synth.normal_bf16((rows, cols), std, seed)
    w = synth.with_outlier_columns(w, synth.outlier_columns(cols, 0.05, seed + 1))
    return w, synth.lognormal((cols,), seed + 2)


def _payload_d(p):
    return np.ascontiguousarray(p[..., 0:2]).view(np.uint16)[..., 0]


def _pow2_d(p):
    """fp16 bits of the power of two nearest (in log) to every block's d."""
    d = _payload_d(p).view(np.float16).astype(np.float64)
    e = np.round(np.log2(d))
    return np.exp2(e).astype(np.float16).view(np.uint16)


def _set_d(p, bits):
    q = p.copy()
    q[..., 0] = (bits & 0xFF).astype(np.uint8)
    q[..., 1] = (bits >> 8).astype(np.uint8)
    return q


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("mode", ["search", "fixed", "every"])
def test_given_predicted_d_reproduces_the_payload(grids, anchors, fmt, mode):
    w, imp = _case(6, 768, 71)
    G = 8 if fmt == "iq1_s" else 16
    kw = {}
    if mode == "fixed":
        kw["choices"] = np.random.default_rng(72).integers(0, 16, (6, 3, G), dtype=np.uint8)
    if mode == "every":
        kw["every_choice"] = True
    p, f = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, **kw)
    assert f == 0
    d = _payload_d(p[0] if mode == "every" else p)
    q, f2 = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, scales=d, **kw)
    assert f2 == 0
    np.testing.assert_array_equal(q, p)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("weighted", [False, True])
def test_decoding_reencodes_to_zero_error_under_its_scales(grids, anchors, fmt, weighted):
    w, imp = _case(8, 1024, 81)
    if not weighted:
        imp = None
    p, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    d2 = _pow2_d(p)
    pin = _set_d(p, d2)
    xhat = oracle.decode(fmt, grids[fmt], pin)                 # fp32, exact
    xb = torch.from_numpy(xhat).reshape(8, 1024).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(xhat).reshape(8, 1024))  # bf16 holds it exactly
    q, f = oracle.encode(fmt, grids[fmt], anchors[fmt], xb, importance=imp, scales=d2)
    assert f == 0
    np.testing.assert_array_equal(oracle.decode(fmt, grids[fmt], q), xhat)
    # no two codes of these grids decode to the same 8 values here, so the pin is byte-exact
    np.testing.assert_array_equal(q, pin)


def _iq1s_check_under(x, w, grid, p, d_given):
    d, ls, neg, idx = iq1s_fields(p)
    assert d == d_given
    chosen = ls + 8 * neg
    for k in range(8):
        objs = [iq1s_group_objectives(x[32 * k + 8 * i:32 * k + 8 * i + 8],
                                      w[32 * k + 8 * i:32 * k + 8 * i + 8], grid, d) for i in range(4)]
        per_c = sum(o.min(axis=1) for o in objs)
        got = sum(objs[i][chosen[k], idx[4 * k + i]] for i in range(4))
        assert got <= per_c.min() * (1 + 2e-5) + 1e-30, (k, got, per_c.min())


def _iq2xs_check_under(x, w, grid, p, d_given):
    d, ls, idx, s7 = iq2xs_fields(p)
    assert d == d_given
    signs = iq2xs_signs(s7)
    for k in range(16):
        objs = [iq2xs_group_objectives(x[16 * k + 8 * i:16 * k + 8 * i + 8], w[16 * k + 8 * i:16 * k + 8 * i + 8],
                                       signs[2 * k + i], grid, d) for i in range(2)]
        per_ls = objs[0].min(1) + objs[1].min(1)
        got = objs[0][ls[k], idx[2 * k]] + objs[1][ls[k], idx[2 * k + 1]]
        assert got <= per_ls.min() * (1 + 2e-5) + 1e-30, (k, got, per_ls.min())


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("factor", [0.37, 1.9])
def test_search_under_a_foreign_d_reaches_bruteforce_minimum(grids, anchors, fmt, factor):
    w, imp = _case(3, 768, 91)
    p0, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    d = (_payload_d(p0).view(np.float16).astype(np.float32) * factor).astype(np.float16).view(np.uint16)
    p, f = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, scales=d)
    assert f == 0
    x = w.double().numpy().reshape(3, 3, 256)
    wi = imp.double().numpy().reshape(3, 256)
    check = _iq1s_check_under if fmt == "iq1_s" else _iq2xs_check_under
    for r in range(3):
        for b in range(3):
            check(x[r, b], wi[b], grids[fmt], p[r, b], float(d[r, b:b + 1].view(np.float16)[0]))


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_static_scale_policy(grids, anchors, fmt):
    w, imp = _case(2, 2048, 101)
    w[1, 256:512] = 0.0                               # an all-zero block that still gets a d
    p0, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    d = _payload_d(p0).copy()
    d[1, 1] = 0x3C00                                  # 1.0 for the zero block
    bad = {0: 0xBC00, 1: 0x7C00, 2: 0xFC00, 3: 0x7E00}  # -1, +inf, -inf, NaN
    for b, h in bad.items():
        d[0, b] = h
    d[0, 4] = 0x8000                                  # -0: zero payload, no finding
    d[0, 5] = 0x0000
    d[0, 6] = 0x0001                                  # the smallest subnormal is a valid scale
    p, f = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, scales=d)
    assert f == FLAG_RANGE
    for b in range(6):
        assert not p[0, b].any(), b
    assert p[0, 6, 0] == 1 and p[0, 6, 1] == 0 and p[0, 6, 2:].any()
    np.testing.assert_array_equal(p[0, 7], p0[0, 7])  # untouched blocks stay as predicted
    # the zero block is searched under d = 1: least sum w xhat^2
    z = p[1, 1]
    assert z[0] == 0x00 and z[1] == 0x3C
    wi = imp.double().numpy()[256:512]
    check = _iq1s_check_under if fmt == "iq1_s" else _iq2xs_check_under
    check(np.zeros(256), wi, grids[fmt], z, 1.0)
    # a refused d is reported together with the block's other findings
    w2 = w.clone()
    w2[0, 0] = float("nan")
    _, f2 = oracle.encode(fmt, grids[fmt], anchors[fmt], w2, importance=imp, scales=d)
    assert f2 == FLAG_RANGE | 1


def test_every_choice_under_scales_matches_fixed(grids, anchors):
    for fmt, G in (("iq1_s", 8), ("iq2_xs", 16)):
        w, imp = _case(2, 512, 111)
        d = np.full((2, 2), 0x1C00, dtype=np.uint16)  # 2^-8
        every, f = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True, scales=d)
        assert f == 0
        for c in (0, 5, 15):
            fixed, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp,
                                     choices=np.full((2, 2, G), c, np.uint8), scales=d)
            np.testing.assert_array_equal(every[c], fixed)
