"""Static-scale encode (PR #3197 "Static scales"): CUDA path vs the CPU oracle, bit for bit.

Scales are given as a dense fp16 array or read in place from an existing payload's d fields,
in every encode mode, batched, with refused and degenerate scales mixed in; at full size the
re-encode of a weight under its own payload's scales must reproduce that payload.
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
def descs(dev, grids, anchors):
    return {fmt: iq.make_desc(fmt, torch.from_numpy(grids[fmt]).to(dev), anchors[fmt])
            for fmt in ("iq1_s", "iq2_xs")}


def _case(shape, seed, std=0.02):
    w = synth.normal_bf16(shape, std, seed)
    w = synth.with_outlier_columns(w, synth.outlier_columns(shape[-1], 0.03, seed + 1))
    ishape = (shape[-1],) if len(shape) == 2 else (shape[0], shape[-1])
    return w, synth.lognormal(ishape, seed + 2)


def _scales(w, fmt, grids, anchors, imp, seed):
    """Predicted d times a factor in [0.5, 2), with refused and degenerate scales mixed in."""
    if w.dim() == 3:
        p = np.stack([oracle.encode(fmt, grids[fmt], anchors[fmt], w[e], importance=imp[e])[0]
                      for e in range(w.shape[0])])
    else:
        p = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)[0]
    d = np.ascontiguousarray(p[..., 0:2]).view(np.uint16)[..., 0].view(np.float16).astype(np.float32)
    rng = np.random.default_rng(seed)
    d = (d * rng.uniform(0.5, 2.0, d.shape)).astype(np.float16).view(np.uint16)
    flat = d.reshape(-1)
    special = [0xBC00, 0x7C00, 0xFC00, 0x7E00, 0x8000, 0x0000, 0x0001, 0x3C00]
    pos = rng.choice(flat.size, size=min(len(special), flat.size // 4), replace=False)
    for i, k in enumerate(pos):
        flat[k] = special[i]
    return d


def _oracle_batched(fmt, grids, anchors, w, imp, scales, **kw):
    if w.dim() == 2:
        return oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, scales=scales, **kw)
    outs, f = [], 0
    for e in range(w.shape[0]):
        ch = kw.get("choices")
        kwe = dict(kw, choices=None if ch is None else ch[e])
        o, fe = oracle.encode(fmt, grids[fmt], anchors[fmt], w[e], importance=imp[e], scales=scales[e], **kwe)
        outs.append(o)
        f |= fe
    axis = 1 if kw.get("every_choice") else 0
    return np.stack(outs, axis=axis), f


def _run(dev, desc, w, imp, scales_t, **kw):
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    p = iq.iq_encode(desc, w.to(dev), imp.to(dev), flags=flags, raise_on_flags=False, scales=scales_t, **kw)
    torch.cuda.synchronize()
    return p.cpu().numpy(), int(flags.item())


def _assert_same(got, want):
    mism = np.nonzero((got != want).any(-1))
    assert not len(mism[0]), f"{len(mism[0])} blocks differ, first {list(zip(*mism))[:5]}"


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("mode", ["search", "fixed", "every"])
@pytest.mark.parametrize("shape", [(37, 768), (3, 21, 512)])
def test_dense_scales_match_oracle(dev, descs, grids, anchors, fmt, mode, shape):
    w, imp = _case(shape, 400 + len(shape), std=0.02 if fmt == "iq1_s" else 0.015)
    d = _scales(w, fmt, grids, anchors, imp, 401)
    kw = {}
    if mode == "fixed":
        kw["choices"] = np.random.default_rng(402).integers(0, 16, d.shape + (iq.CHOICE_GROUPS[fmt],),
                                                             dtype=np.uint8)
    if mode == "every":
        kw["every_choice"] = True
    want, wf = _oracle_batched(fmt, grids, anchors, w, imp, d, **kw)
    gkw = dict(kw)
    if "choices" in gkw:
        gkw["choices"] = torch.from_numpy(gkw["choices"]).to(dev)
    got, gf = _run(dev, descs[fmt], w, imp, torch.from_numpy(d.view(np.float16)).to(dev), **gkw)
    assert wf == gf and (gf & iq.FLAG_RANGE)
    _assert_same(got, want)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_scales_read_in_place_from_a_payload(dev, descs, grids, anchors, fmt):
    w, imp = _case((53, 1024), 410)
    d = _scales(w, fmt, grids, anchors, imp, 411)
    holder = np.zeros(d.shape + (iq.BLOCK_BYTES[fmt],), np.uint8)
    holder[..., 0] = (d & 0xFF).astype(np.uint8)
    holder[..., 1] = (d >> 8).astype(np.uint8)
    holder[..., 2:] = 0xA5                             # the rest of the payload is not read
    want, wf = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, scales=d)
    got, gf = _run(dev, descs[fmt], w, imp, torch.from_numpy(holder).to(dev))
    assert wf == gf
    _assert_same(got, want)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_decoding_reencodes_to_the_pin(dev, descs, grids, anchors, fmt):
    """GPU decode (bf16) of a payload with power-of-two d, re-encoded under that payload in place."""
    w, imp = _case((64, 2048), 420)
    p, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    d = np.ascontiguousarray(p[..., 0:2]).view(np.uint16)[..., 0].view(np.float16).astype(np.float64)
    d2 = np.exp2(np.round(np.log2(d))).astype(np.float16).view(np.uint16)
    pin = p.copy()
    pin[..., 0] = (d2 & 0xFF).astype(np.uint8)
    pin[..., 1] = (d2 >> 8).astype(np.uint8)
    pin_d = torch.from_numpy(pin).to(dev)
    xb = iq.iq_decode(descs[fmt], pin_d, torch.bfloat16).reshape(64, 2048)
    xf = torch.from_numpy(oracle.decode(fmt, grids[fmt], pin)).reshape(64, 2048)
    assert torch.equal(xb.float().cpu(), xf)
    got = iq.iq_encode(descs[fmt], xb, imp.to(dev), scales=pin_d).cpu().numpy()
    _assert_same(got, pin)


def test_full_size_reencode_under_own_scales(dev, descs):
    """4096 x 4096 IQ1_S weight, importance-weighted: the encode under its own payload's d
    (read in place) reproduces the payload; sampled rows also match the oracle."""
    wl = synth.workload_iq1s_4096x4096_weighted()
    w, imp = wl["w"].to(dev), wl["importance"].to(dev)
    p = iq.iq_encode(descs["iq1_s"], w, imp)
    q = iq.iq_encode(descs["iq1_s"], w, imp, scales=p)
    assert torch.equal(p, q)
    d16 = p[..., 0:2].contiguous().view(torch.float16).reshape(4096, 16)
    half = (d16.float() * 0.75).half().contiguous()
    r = iq.iq_encode(descs["iq1_s"], w, imp, scales=half)
    rows = np.random.default_rng(430).choice(4096, 6, replace=False)
    grid = synth.iq1s_grid()
    for row in rows:
        want, _ = oracle.encode("iq1_s", grid, 0.61, wl["w"][row:row + 1], importance=wl["importance"],
                                scales=half[row:row + 1].cpu().numpy())
        _assert_same(r[row:row + 1].cpu().numpy(), want)


def test_bad_scales_arguments(dev, descs):
    w = torch.zeros((4, 512), dtype=torch.bfloat16, device=dev)
    with pytest.raises(iq.IQError):
        iq.iq_encode(descs["iq1_s"], w, scales=torch.zeros(7, dtype=torch.float16, device=dev))
    with pytest.raises(iq.IQError):
        iq.iq_encode(descs["iq1_s"], w, scales=torch.zeros((4, 2, 74), dtype=torch.uint8, device=dev))
