"""Pins of the oracle's fp32 and f16 weight inputs (CPU only, no GPU).

PR #2450's encoders take fp32, f16 and bf16 weights; each converts to fp32 exactly, and the search
runs on those fp32 values. What fixes the oracle here:

* fp64 brute force on fp32 weights that bf16 cannot hold, for every format;
* the same values given as bf16, f16 or fp32 encode to the same payload;
* the static-scale round trip without the power-of-two restriction: an fp32 decode is exact, so
  the decoding of any payload re-encodes, under that payload's scales, to the payload itself;
* non-finite fp32 weights are refused like bf16 ones.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from fp64_refs import (iq1m_fields, iq1s_fields, iq1s_group_objectives, iq2s_fields, iq2xs_fields,
                       iq2xs_group_objectives, iq2xs_signs, signs_of_mask)
from ggml_iq_codebook_b200 import synth

FMTS = ["iq1_s", "iq2_xs", "iq1_m", "iq2_s"]


def _f32_case(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((rows, cols), generator=g) * 0.02
    x[:, ::37] *= 8.0
    return x, synth.lognormal((cols,), seed + 1)


def _d(fmt, p):
    return {"iq1_s": iq1s_fields, "iq2_xs": iq2xs_fields, "iq1_m": iq1m_fields, "iq2_s": iq2s_fields}[fmt](p)[0]


def _check(fmt, grid, x, w, p):
    """Every choice group's pick reaches the fp64 minimum of sum w (x - xhat)^2 over its options."""
    if fmt in ("iq1_s", "iq1_m"):
        if fmt == "iq1_s":
            d, ls, neg, idx = iq1s_fields(p)
            span, per = 32, 4
            choice = lambda k, i: ls[k] + 8 * neg[k]             # noqa: E731
        else:
            d, ls, neg, idx = iq1m_fields(p)
            span, per = 16, 2
            choice = lambda k, i: ls[k] + 8 * neg[per * k + i]   # noqa: E731
        for k in range(256 // span):
            objs = [iq1s_group_objectives(x[span * k + 8 * i:span * k + 8 * i + 8], w[span * k + 8 * i:span * k + 8 * i + 8],
                                          grid, d) for i in range(per)]
            if fmt == "iq1_s":
                best = min(sum(o[c].min() for o in objs) for c in range(16))
            else:
                best = min(sum(min(o[l].min(), o[l + 8].min()) for o in objs) for l in range(8))
            got = sum(objs[i][choice(k, i), idx[per * k + i]] for i in range(per))
            scale = float((w[span * k:span * k + span] * x[span * k:span * k + span] ** 2).sum())
            assert got <= best + 2e-5 * scale, (fmt, k)
    else:
        if fmt == "iq2_xs":
            d, ls, idx, s7 = iq2xs_fields(p)
            signs = iq2xs_signs(s7)
        else:
            d, ls, idx, s8 = iq2s_fields(p)
            signs = signs_of_mask(s8)
        for k in range(16):
            objs = [iq2xs_group_objectives(x[16 * k + 8 * i:16 * k + 8 * i + 8], w[16 * k + 8 * i:16 * k + 8 * i + 8],
                                           signs[2 * k + i], grid, d) for i in range(2)]
            per_ls = objs[0].min(1) + objs[1].min(1)
            got = objs[0][ls[k], idx[2 * k]] + objs[1][ls[k], idx[2 * k + 1]]
            scale = float((w[16 * k:16 * k + 16] * x[16 * k:16 * k + 16] ** 2).sum())
            assert got <= per_ls.min() + 2e-5 * scale, (fmt, k)


@pytest.mark.parametrize("fmt", FMTS)
def test_fp32_search_reaches_bruteforce_minimum(grids, anchors, fmt):
    x, imp = _f32_case(2, 512, 301)
    assert not torch.equal(x.bfloat16().float(), x)            # values bf16 cannot hold
    p, f = oracle.encode(fmt, grids[fmt], anchors[fmt], x, importance=imp)
    assert f == 0
    xd, wd = x.double().numpy(), imp.double().numpy()
    for r in range(2):
        for b in range(2):
            _check(fmt, grids[fmt], xd[r, 256 * b:256 * b + 256], wd[256 * b:256 * b + 256], p[r, b])


@pytest.mark.parametrize("fmt", FMTS)
def test_input_kinds_agree_on_equal_values(grids, anchors, fmt):
    x, imp = _f32_case(4, 512, 311)
    h = x.half()                                                # f16 values, exactly representable in fp32
    ph, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], h, importance=imp)
    pf, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], h.float(), importance=imp)
    np.testing.assert_array_equal(ph, pf)
    b = x.bfloat16()
    pb, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], b, importance=imp)
    pf2, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], b.float().numpy(), importance=imp)
    np.testing.assert_array_equal(pb, pf2)
    assert not np.array_equal(ph, pb)                          # the inputs do differ


@pytest.mark.parametrize("fmt", FMTS)
def test_fp32_decoding_reencodes_to_the_payload_under_its_scales(grids, anchors, fmt):
    x, imp = _f32_case(6, 1024, 321)
    p, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], x, importance=imp)
    d = np.array([[_d(fmt, blk) for blk in row] for row in p], np.float64).astype(np.float16)
    xhat = oracle.decode(fmt, grids[fmt], p).reshape(6, 1024)  # exact in fp32
    q, f = oracle.encode(fmt, grids[fmt], anchors[fmt], xhat, importance=imp, scales=d)
    assert f == 0
    np.testing.assert_array_equal(q, p)


def test_nonfinite_fp32_is_refused(grids, anchors):
    x, imp = _f32_case(3, 256, 331)
    x[1, 7] = float("nan")
    x[2, 9] = float("-inf")
    p, f = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], x, importance=imp)
    assert f == 1 and not p[1].any() and not p[2].any() and p[0].any()
