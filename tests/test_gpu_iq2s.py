"""IQ2_S (PR #2512 codec, PR #2565 CUDA encoder): CUDA path vs the CPU oracle, bit for bit.

Search, fixed and every-choice encodes over sizes that span several persistent-CTA strides and
ragged tails, batched and strided inputs, static scales (dense and read in place from a payload),
the flag policy, the decode of random payloads (fp32 and bf16), and an 8192 x 4096 weight with the
oracle on sampled rows.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq
import oracle
from ggml_iq_codebook_b200 import build, synth

pytestmark = pytest.mark.gpu
B = 82
ANCHOR = 0.9


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    iq.load_library()
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def grid():
    return synth.iq2s_grid()


@pytest.fixture(scope="module")
def desc(dev, grid):
    return iq.make_desc("iq2_s", torch.from_numpy(grid).to(dev), ANCHOR)


def _case(shape, seed, std=0.015, weighted=True):
    w = synth.normal_bf16(shape, std, seed)
    w = synth.with_outlier_columns(w, synth.outlier_columns(shape[-1], 0.03, seed + 1))
    ishape = (shape[-1],) if len(shape) == 2 else (shape[0], shape[-1])
    return w, (synth.lognormal(ishape, seed + 2) if weighted else None)


def _gpu(desc, w, imp, dev, **kw):
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    p = iq.iq_encode(desc, w.to(dev), None if imp is None else imp.to(dev), flags=flags, raise_on_flags=False, **kw)
    torch.cuda.synchronize()
    return p.cpu().numpy(), int(flags.item())


def _same(got, want):
    mism = np.nonzero((got != want).any(-1))
    assert not len(mism[0]), f"{len(mism[0])} blocks differ, first {list(zip(*mism))[:5]}"


@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("rows,cols", [(1, 256), (37, 768), (160, 4096)])
def test_search_matches_oracle(dev, desc, grid, weighted, rows, cols):
    w, imp = _case((rows, cols), 700 + rows, weighted=weighted)
    got, gf = _gpu(desc, w, imp, dev)
    want, wf = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp)
    assert gf == wf == 0
    _same(got, want)


def test_fixed_choices_match_oracle(dev, desc, grid):
    w, imp = _case((29, 768), 710)
    ch = np.random.default_rng(711).integers(0, 16, size=(29, 3, 16)).astype(np.uint8)
    got, gf = _gpu(desc, w, imp, dev, choices=torch.from_numpy(ch).to(dev))
    want, wf = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp, choices=ch)
    assert gf == wf == 0
    _same(got, want)
    ch[3, 1, 9] = 16
    got, gf = _gpu(desc, w, imp, dev, choices=torch.from_numpy(ch).to(dev))
    assert gf == iq.FLAG_CHOICE and not got[3, 1].any()


def test_every_choice_matches_oracle(dev, desc, grid):
    w, imp = _case((11, 512), 720)
    got, gf = _gpu(desc, w, imp, dev, every_choice=True)
    want, wf = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp, every_choice=True)
    assert gf == wf == 0 and got.shape == (16, 11, 2, B)
    _same(got, want)
    for c in (0, 9, 15):
        forced, _ = _gpu(desc, w, imp, dev, choices=torch.full((11, 2, 16), c, dtype=torch.uint8, device=dev))
        assert np.array_equal(forced, got[c])


def test_batched_and_strided(dev, desc, grid):
    w, imp = _case((4, 5, 512), 730)
    got, gf = _gpu(desc, w, imp, dev)
    assert gf == 0 and got.shape == (4, 5, 2, B)
    for e in range(4):
        want, _ = oracle.encode("iq2_s", grid, ANCHOR, w[e], importance=imp[e])
        _same(got[e], want)
    big, imp2 = _case((9, 1024), 731)
    view = big.to(dev)[:, 256:768]
    got = iq.iq_encode(desc, view, imp2[256:768].to(dev).contiguous()).cpu().numpy()
    want, _ = oracle.encode("iq2_s", grid, ANCHOR, big[:, 256:768].contiguous(), importance=imp2[256:768])
    _same(got, want)


@pytest.mark.parametrize("mode", ["search", "fixed", "every"])
def test_static_scales_match_oracle(dev, desc, grid, mode):
    w, imp = _case((23, 768), 740)
    p0, _ = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp)
    d = (np.ascontiguousarray(p0[..., 0:2]).view(np.float16)[..., 0].astype(np.float32) *
         np.random.default_rng(741).uniform(0.5, 2.0, p0.shape[:2])).astype(np.float16).view(np.uint16)
    d[0, 0], d[1, 1], d[2, 2], d[3, 0], d[4, 1] = 0xBC00, 0x7C00, 0x7E00, 0x8000, 0x0001
    kw = {}
    if mode == "fixed":
        kw["choices"] = np.random.default_rng(742).integers(0, 16, (23, 3, 16), dtype=np.uint8)
    if mode == "every":
        kw["every_choice"] = True
    want, wf = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp, scales=d, **kw)
    gkw = dict(kw)
    if "choices" in gkw:
        gkw["choices"] = torch.from_numpy(gkw["choices"]).to(dev)
    got, gf = _gpu(desc, w, imp, dev, scales=torch.from_numpy(d.view(np.float16)).to(dev), **gkw)
    assert gf == wf == iq.FLAG_RANGE
    _same(got, want)
    if mode == "search":                              # the same d read in place from a payload
        holder = np.full(p0.shape, 0x5A, np.uint8)
        holder[..., 0] = (d & 0xFF).astype(np.uint8)
        holder[..., 1] = (d >> 8).astype(np.uint8)
        got2, _ = _gpu(desc, w, imp, dev, scales=torch.from_numpy(holder).to(dev))
        _same(got2, want)


def test_zero_nonfinite_range_policy(dev, desc, grid):
    w, imp = _case((6, 256), 750)
    w = w.clone()
    w[1] = 0.0
    w[2] = 1e-7
    w[3, 17] = float("nan")
    w[4, 5] = float("inf")
    w[5, 0] = 3e9
    got, gf = _gpu(desc, w, imp, dev)
    want, wf = oracle.encode("iq2_s", grid, ANCHOR, w, importance=imp)
    assert gf == wf == (iq.FLAG_NONFINITE | iq.FLAG_RANGE)
    _same(got, want)
    g = grid.copy()
    g[5, 3] = 2
    bad = iq.make_desc("iq2_s", torch.from_numpy(g).to(dev), ANCHOR)
    got, gf = _gpu(bad, w[:1], imp, dev)
    assert gf & iq.FLAG_GRID and not got.any()


def _random_payload(nblocks, seed):
    rng = np.random.default_rng(seed)
    p = rng.integers(0, 256, size=(nblocks, B), dtype=np.uint8)
    d = rng.uniform(1e-4, 3.0, size=nblocks).astype(np.float16).view(np.uint16)
    p[:, 0] = d & 0xFF
    p[:, 1] = d >> 8
    return p


@pytest.mark.parametrize("nblocks", [1, 31, 33, 1000, 4099])
def test_decode_matches_oracle(dev, desc, grid, nblocks):
    p = _random_payload(nblocks, 760 + nblocks)
    want = oracle.decode("iq2_s", grid, p)
    pd = torch.from_numpy(p).to(dev)
    got32 = iq.iq_decode(desc, pd, torch.float32).cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    got16 = iq.iq_decode(desc, pd, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got16, oracle.f32_to_bf16_bits(want))


def test_full_size_8192x4096(dev, desc, grid):
    wl = synth.workload_iq2xs_8192x4096()
    got = iq.iq_encode(desc, wl["w"].to(dev), wl["importance"].to(dev)).cpu().numpy()
    rows = np.random.default_rng(770).choice(8192, 6, replace=False)
    for r in rows:
        want, _ = oracle.encode("iq2_s", grid, ANCHOR, wl["w"][r:r + 1], importance=wl["importance"])
        _same(got[r:r + 1], want)
