"""CUDA path vs the CPU oracle, bit for bit, through the C ABI (needs a B200).

Small cases span several CTA strides and ragged tails; the five workloads run at full size in the
launch configuration bench.py times, with the oracle recomputing sampled rows.
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
    out = {}
    for fmt in ("iq1_s", "iq2_xs", "iq2_s"):
        g = torch.from_numpy(grids[fmt]).to(dev)
        out[fmt] = iq.make_desc(fmt, g, anchors[fmt])
    return out


def _case(rows, cols, seed, std=0.02, outlier_frac=0.02, weighted=True, batch=None):
    shape = (rows, cols) if batch is None else (batch, rows, cols)
    w = synth.normal_bf16(shape, std, seed)
    if outlier_frac:
        w = synth.with_outlier_columns(w, synth.outlier_columns(cols, outlier_frac, seed + 1))
    ishape = (cols,) if batch is None else (batch, cols)
    imp = synth.lognormal(ishape, seed + 2) if weighted else None
    return w, imp


def _gpu_encode(desc, w, imp, dev, **kw):
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    p = iq.iq_encode(desc, w.to(dev), None if imp is None else imp.to(dev), flags=flags,
                     raise_on_flags=False, **kw)
    torch.cuda.synchronize()
    return p.cpu().numpy(), int(flags.item())


# --------------------------------------------------------------------------------- encode parity

@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("rows,cols", [(1, 256), (37, 768), (160, 4096)])
def test_encode_search_matches_oracle(dev, descs, grids, anchors, fmt, weighted, rows, cols):
    w, imp = _case(rows, cols, 200 + rows, std=0.02 if fmt == "iq1_s" else 0.015, weighted=weighted)
    got, gf = _gpu_encode(descs[fmt], w, imp, dev)
    want, wf = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    assert gf == wf == 0
    mism = np.nonzero((got != want).any(-1))
    assert not len(mism[0]), f"{len(mism[0])} blocks differ, first {list(zip(*mism))[:5]}"


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_encode_fixed_choices_match_oracle(dev, descs, grids, anchors, fmt):
    G = iq.CHOICE_GROUPS[fmt]
    w, imp = _case(29, 768, 301)
    ch = np.random.default_rng(7).integers(0, 16, size=(29, 3, G)).astype(np.uint8)
    got, gf = _gpu_encode(descs[fmt], w, imp, dev, choices=torch.from_numpy(ch).to(dev))
    want, wf = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, choices=ch)
    assert gf == wf == 0
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_encode_every_choice_matches_oracle(dev, descs, grids, anchors, fmt):
    """PR #3159: payload c == forced encode with choices = full(c), from one sweep."""
    w, imp = _case(11, 512, 311)
    got, gf = _gpu_encode(descs[fmt], w, imp, dev, every_choice=True)
    want, wf = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    assert gf == wf == 0
    assert got.shape == (16, 11, 2, iq.BLOCK_BYTES[fmt])
    assert np.array_equal(got, want)
    # and against the GPU's own forced encodes
    for c in (0, 7, 8, 15):
        full = torch.full((11, 2, iq.CHOICE_GROUPS[fmt]), c, dtype=torch.uint8, device=dev)
        forced, _ = _gpu_encode(descs[fmt], w, imp, dev, choices=full)
        assert np.array_equal(forced, got[c])


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_encode_batched_matches_per_expert_oracle(dev, descs, grids, anchors, fmt):
    w, imp = _case(5, 512, 321, batch=4)
    got, gf = _gpu_encode(descs[fmt], w, imp, dev)
    assert gf == 0 and got.shape == (4, 5, 2, iq.BLOCK_BYTES[fmt])
    for e in range(4):
        want, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w[e], importance=imp[e])
        assert np.array_equal(got[e], want), e
    # one importance vector shared by every expert (batch stride 0)
    got_s, _ = _gpu_encode(descs[fmt], w, imp[1], dev)
    want_s, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w[2], importance=imp[1])
    assert np.array_equal(got_s[2], want_s)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_encode_strided_rows(dev, descs, grids, anchors, fmt):
    big, imp = _case(9, 1024, 331)
    view = big.to(dev)[:, 256:768]  # ldw = 1024, 2 blocks per row
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    got = iq.iq_encode(descs[fmt], view, imp[256:768].to(dev).contiguous(), flags=flags).cpu().numpy()
    want, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], big[:, 256:768].contiguous(), importance=imp[256:768])
    assert np.array_equal(got, want)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_uniform_power_of_two_importance_is_the_unweighted_payload(dev, descs, fmt):
    w, _ = _case(16, 512, 341, weighted=False)
    p0, _ = _gpu_encode(descs[fmt], w, None, dev)
    for c in (1.0, 2.0, 0.25):
        p1, _ = _gpu_encode(descs[fmt], w, torch.full((512,), c), dev)
        assert np.array_equal(p0, p1)


def test_encode_is_deterministic(dev, descs):
    w, imp = _case(64, 1024, 351)
    a, _ = _gpu_encode(descs["iq1_s"], w, imp, dev)
    b, _ = _gpu_encode(descs["iq1_s"], w, imp, dev)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_zero_nonfinite_range_and_choice_policy(dev, descs, grids, anchors, fmt):
    w, imp = _case(6, 256, 361)
    w = w.clone()
    w[1] = 0.0
    w[2] = 1e-7
    w[3, 17] = float("nan")
    w[4, 5] = float("inf")
    w[5, 0] = 3e9
    got, gf = _gpu_encode(descs[fmt], w, imp, dev)
    want, wf = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp)
    assert gf == wf == (iq.FLAG_NONFINITE | iq.FLAG_RANGE)
    assert np.array_equal(got, want)
    with pytest.raises(iq.IQError) as ei:
        iq.iq_encode(descs[fmt], w.to(dev), imp.to(dev))
    assert ei.value.flags == gf
    bad = imp.clone()
    bad[3] = -1.0
    got, gf = _gpu_encode(descs[fmt], w[:1], bad, dev)
    assert gf == iq.FLAG_IMPORTANCE and not got.any()
    bad[3] = float("inf")
    got, gf = _gpu_encode(descs[fmt], w[:1], bad, dev)
    assert gf == iq.FLAG_IMPORTANCE and not got.any()
    ch = torch.full((1, 1, iq.CHOICE_GROUPS[fmt]), 16, dtype=torch.uint8, device=dev)
    got, gf = _gpu_encode(descs[fmt], w[:1], imp, dev, choices=ch)
    assert gf == iq.FLAG_CHOICE and not got.any()


def test_bad_grid_is_flagged(dev, grids, anchors):
    g = grids["iq1_s"].copy()
    g[5, 3] = 2
    desc = iq.make_desc("iq1_s", torch.from_numpy(g).to(dev), anchors["iq1_s"])
    w, imp = _case(2, 256, 371)
    got, gf = _gpu_encode(desc, w, imp, dev)
    assert gf & iq.FLAG_GRID and not got.any()


def test_wrong_shapes_raise(dev, descs):
    with pytest.raises(iq.IQError):
        iq.iq_encode(descs["iq1_s"], torch.zeros((512, 384), dtype=torch.bfloat16, device=dev))
    with pytest.raises(iq.IQError):
        iq.iq_encode(descs["iq1_s"], torch.zeros((0, 256), dtype=torch.bfloat16, device=dev))
    with pytest.raises(iq.IQError):
        iq.iq_encode(descs["iq1_s"], torch.zeros((4, 256), dtype=torch.float64, device=dev))


# --------------------------------------------------------------------------------- decode parity

def _random_payload(fmt, nblocks, seed):
    rng = np.random.default_rng(seed)
    p = rng.integers(0, 256, size=(nblocks, iq.BLOCK_BYTES[fmt]), dtype=np.uint8)
    d = rng.uniform(1e-4, 3.0, size=nblocks).astype(np.float16).view(np.uint16)  # finite d
    p[:, 0] = d & 0xFF
    p[:, 1] = d >> 8
    return p


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
@pytest.mark.parametrize("nblocks", [1, 31, 33, 1000, 4099])
def test_decode_matches_oracle(dev, descs, grids, fmt, nblocks):
    p = _random_payload(fmt, nblocks, 400 + nblocks)
    want = oracle.decode(fmt, grids[fmt], p)
    pd = torch.from_numpy(p).to(dev)
    got32 = iq.iq_decode(descs[fmt], pd, torch.float32).cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), want.view(np.uint32))
    got16 = iq.iq_decode(descs[fmt], pd, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got16, oracle.f32_to_bf16_bits(want))


@pytest.mark.parametrize("fmt", ["iq1_s", "iq2_xs"])
def test_decode_is_chunk_invariant(dev, descs, fmt):
    p = torch.from_numpy(_random_payload(fmt, 777, 451)).to(dev)
    whole = iq.iq_decode(descs[fmt], p, torch.bfloat16)
    parts = torch.cat([iq.iq_decode(descs[fmt], p[a:b].contiguous(), torch.bfloat16)
                       for a, b in ((0, 1), (1, 100), (100, 101), (101, 777))])
    assert torch.equal(whole, parts)


def test_decode_of_unaligned_payload_view(dev, descs, grids):
    p = _random_payload("iq1_s", 65, 461)
    pd = torch.from_numpy(p).to(dev)[1:].contiguous()
    raw = torch.empty(64 * 50 + 2, dtype=torch.uint8, device=dev)
    view = raw[2:].view(64, 50)  # start 2 bytes past a 16-byte boundary
    view.copy_(pd)
    got = iq.iq_decode(descs["iq1_s"], view, torch.float32).cpu().numpy()
    assert np.array_equal(got, oracle.decode("iq1_s", grids["iq1_s"], p[1:]))


# --------------------------------------------------------------------------------- choice search

def _choice_case(fmt, rows, nblk, seed, offdiag):
    w = synth.normal_bf16((rows, nblk * 256), 0.02, seed)
    hess = torch.stack([synth.block_hessian(seed + 10 + b, offdiag_std=offdiag) for b in range(nblk)])
    return w, hess


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s"])
@pytest.mark.parametrize("offdiag", [0.02, 0.3])
def test_choice_search_matches_oracle(dev, descs, grids, anchors, fmt, offdiag):
    rows, nblk = 13, 2
    w, hess = _choice_case(fmt, rows, nblk, 501, offdiag)
    imp = oracle.sqrt_diag(hess.numpy())
    cand, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    want_p, want_pay = oracle.choice_search(fmt, grids[fmt], w, hess.numpy(), cand)
    picks, pay = iq.iq_choice_search(descs[fmt], w.to(dev), hess.to(dev), torch.from_numpy(cand).to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(picks.cpu().numpy(), want_p)
    assert np.array_equal(pay.cpu().numpy(), want_pay)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s", "iq1_m", "g8"])
def test_choice_search_exact_ties_match_oracle(dev, grids, anchors, fmt):
    """Candidates duplicated at higher choices (exact ties in every score and gain), and all
    candidates equal: picks, payload and objective bits as the oracle's (the lowest choice wins
    ties, and a zero gain never switches). g8: eight candidates per 8-weight group."""
    efmt = "iq2_xs" if fmt == "g8" else fmt
    desc = iq.make_desc(efmt, torch.from_numpy(grids[efmt]).to(dev), anchors[efmt])
    rows, nblk = 13, 2
    w, hess = _choice_case(efmt, rows, nblk, 521, 0.3)
    imp = oracle.sqrt_diag(hess.numpy())
    cand, _ = oracle.encode(efmt, grids[efmt], anchors[efmt], w, importance=imp, every_choice=True)
    C, lo = cand.shape[0], (8 if fmt == "g8" else 0)
    dup = cand.copy()
    dup[C - 1], dup[lo + 4] = dup[lo + 1], dup[lo + 2]
    same = np.broadcast_to(cand[lo:lo + 1], cand.shape).copy()
    for cd in (dup, same):
        cdev = torch.from_numpy(cd).to(dev)
        obj = torch.empty((rows, nblk), dtype=torch.float32, device=dev)
        if fmt == "g8":
            picks = iq.iq_choice_search_g8(desc, w.to(dev), hess.to(dev), cdev, objective=obj)
            want_p, want_obj = oracle.choice_search_g8(grids["iq2_xs"], w, hess.numpy(), cd, objective=True)
        else:
            picks, pay = iq.iq_choice_search(desc, w.to(dev), hess.to(dev), cdev, objective=obj)
            want_p, want_pay, want_obj = oracle.choice_search(fmt, grids[fmt], w, hess.numpy(), cd, objective=True)
            assert np.array_equal(pay.cpu().numpy(), want_pay)
        assert np.array_equal(picks.cpu().numpy(), want_p)
        assert np.array_equal(obj.cpu().numpy().view(np.uint32), want_obj.view(np.uint32))
        assert not (want_p == C - 1).any() and not (want_p == lo + 4).any()


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s"])
def test_local_hessian_pipeline_on_gpu_matches_oracle(dev, descs, grids, anchors, fmt):
    """sqrt(diag H) -> every-choice encode -> choice search, all in the library's kernels."""
    rows, nblk = 10, 3
    w, hess = _choice_case(fmt, rows, nblk, 511, 0.3)
    hd = hess.to(dev)
    imp_d = iq.iq_sqrt_diag(hd)
    imp = oracle.sqrt_diag(hess.numpy())
    assert np.array_equal(imp_d.cpu().numpy(), imp)
    cand_d = iq.iq_encode(descs[fmt], w.to(dev), imp_d, every_choice=True)
    obj = torch.empty((rows, nblk), dtype=torch.float32, device=dev)
    picks, pay = iq.iq_choice_search(descs[fmt], w.to(dev), hd, cand_d, objective=obj)
    cand, _ = oracle.encode(fmt, grids[fmt], anchors[fmt], w, importance=imp, every_choice=True)
    want_p, want_pay, want_obj = oracle.choice_search(fmt, grids[fmt], w, hess.numpy(), cand, objective=True)
    assert np.array_equal(cand_d.cpu().numpy(), cand)
    assert np.array_equal(picks.cpu().numpy(), want_p)
    assert np.array_equal(pay.cpu().numpy(), want_pay)
    assert np.array_equal(obj.cpu().numpy().view(np.uint32), want_obj.view(np.uint32))  # fp32 bits
    # the final payload is the encode under the picks
    fixed = iq.iq_encode(descs[fmt], w.to(dev), imp_d, choices=picks.contiguous())
    assert torch.equal(fixed, pay)


@pytest.mark.parametrize("fmt", ["iq2_xs", "iq1_s", "iq2_s"])
def test_choice_search_over_a_stack_of_experts(dev, descs, grids, anchors, fmt):
    """Experts of 13 rows (ragged against the 16- and 8-row CTA tiles), each with its own
    Hessian blocks, in one batched encode and one choice-search launch."""
    nexp, rows, nblk = 3, 13, 2
    w = synth.normal_bf16((nexp, rows, nblk * 256), 0.02, 521)
    hess = torch.stack([torch.stack([synth.block_hessian(530 + 10 * e + b, offdiag_std=0.3) for b in range(nblk)])
                        for e in range(nexp)])                        # [E, nblk, 256, 256]
    hd = hess.to(dev)
    imp_d = iq.iq_sqrt_diag(hd).view(nexp, nblk * 256)
    cand_d = iq.iq_encode(descs[fmt], w.to(dev), imp_d, every_choice=True)   # [16, E, rows, nblk, B]
    picks, pay = iq.iq_choice_search(descs[fmt], w.to(dev), hd, cand_d)
    torch.cuda.synchronize()
    imp = oracle.sqrt_diag(hess.numpy()).reshape(nexp, nblk * 256)
    cand = np.stack([oracle.encode(fmt, grids[fmt], anchors[fmt], w[e], importance=imp[e], every_choice=True)[0]
                     for e in range(nexp)], axis=1)
    assert np.array_equal(cand_d.cpu().numpy(), cand)
    want_p, want_pay = oracle.choice_search(fmt, grids[fmt], w, hess.numpy(), cand)
    assert np.array_equal(picks.cpu().numpy(), want_p)
    assert np.array_equal(pay.cpu().numpy(), want_pay)
    for e in range(nexp):                             # and the same as one launch per expert
        pe, ye = iq.iq_choice_search(descs[fmt], w[e].to(dev), hd[e].contiguous(), cand_d[:, e].contiguous())
        assert torch.equal(pe, picks[e]) and torch.equal(ye, pay[e])


def test_choice_search_one_block_per_call(dev, descs, grids, anchors):
    """The same search run as one call per 256-column block, on views into the whole-weight
    tensors (the GPTQ-style calling pattern), gives the picks and payload of one call over all."""
    fmt, rows, nblk = "iq2_xs", 37, 3
    w, hess = _choice_case(fmt, rows, nblk, 541, 0.3)
    wd, hd = w.to(dev), hess.to(dev)
    cand = iq.iq_encode(descs[fmt], wd, iq.iq_sqrt_diag(hd), every_choice=True)
    picks, pay = iq.iq_choice_search(descs[fmt], wd, hd, cand)
    pay_b = torch.zeros_like(pay)
    for b in range(nblk):
        pk, _ = iq.iq_choice_search(descs[fmt], wd[:, 256 * b:256 * (b + 1)], hd[b:b + 1], cand[:, :, b:b + 1],
                                    payload=pay_b[:, b:b + 1])
        assert torch.equal(pk[:, 0], picks[:, b])
    assert torch.equal(pay_b, pay)
    with pytest.raises(iq.IQError):                   # a payload buffer of the wrong shape is refused
        iq.iq_choice_search(descs[fmt], wd, hd, cand, payload=torch.empty((rows, nblk, 73), dtype=torch.uint8,
                                                                          device=dev))


# --------------------------------------------------------------------------------- full sizes

def _sample_rows(rows, k, seed):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(rows, size=k, replace=False).tolist()) | {0, rows - 1}
    return sorted(pick)


def test_full_size_iq1s_4096x4096_weighted(dev, descs, grids, anchors):
    wl = synth.workload_iq1s_4096x4096_weighted()
    got = iq.iq_encode(descs["iq1_s"], wl["w"].to(dev), wl["importance"].to(dev)).cpu().numpy()
    rows = _sample_rows(4096, 6, 601)
    want, _ = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], wl["w"][rows], importance=wl["importance"])
    assert np.array_equal(got[rows], want)


def test_full_size_iq2xs_8192x4096(dev, descs, grids, anchors):
    wl = synth.workload_iq2xs_8192x4096()
    wd = wl["w"].to(dev)
    got = iq.iq_encode(descs["iq2_xs"], wd, wl["importance"].to(dev))
    rows = _sample_rows(8192, 14, 602)
    want, _ = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], wl["w"][rows], importance=wl["importance"])
    assert np.array_equal(got.cpu().numpy()[rows], want)
    dec = iq.iq_decode(descs["iq2_xs"], got, torch.bfloat16)
    want_dec = oracle.f32_to_bf16_bits(oracle.decode("iq2_xs", grids["iq2_xs"], want))
    assert np.array_equal(dec.cpu()[rows].view(torch.int16).numpy().view(np.uint16), want_dec)


def test_full_size_moe_256x1536x4096_one_call(dev, descs, grids, anchors):
    wl = synth.workload_iq1s_moe(device=dev)
    imp = wl["importance"].to(dev)
    got = iq.iq_encode(descs["iq1_s"], wl["w"], imp)
    assert got.shape == (256, 1536, 16, 50)
    rng = np.random.default_rng(603)
    cases = [(e, r) for e in (0, 127, 255) for r in _sample_rows(1536, 2, 604 + e)]
    cases += [(int(e), int(rng.integers(0, 1536))) for e in rng.choice(256, 6, replace=False)]
    for e, r in cases:
        want, _ = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], wl["w"][e, r:r + 1].cpu(),
                                importance=imp[e].cpu())
        assert np.array_equal(got[e, r:r + 1].cpu().numpy(), want), (e, r)
    del got, wl
    torch.cuda.empty_cache()


def test_full_size_choice_search_4096x4096(dev, descs, grids, anchors):
    wl = synth.workload_choice_iq2xs()
    wd, hd = wl["w"].to(dev), wl["hess"].to(dev)
    imp_d = iq.iq_sqrt_diag(hd)
    cand_d = iq.iq_encode(descs["iq2_xs"], wd, imp_d, every_choice=True)
    picks, pay = iq.iq_choice_search(descs["iq2_xs"], wd, hd, cand_d)
    rows = _sample_rows(4096, 3, 605)
    imp = oracle.sqrt_diag(wl["hess"].numpy())
    for r in rows:
        cand, _ = oracle.encode("iq2_xs", grids["iq2_xs"], anchors["iq2_xs"], wl["w"][r:r + 1],
                                importance=imp, every_choice=True)
        assert np.array_equal(cand_d[:, r:r + 1].cpu().numpy(), cand), r
        want_p, want_pay = oracle.choice_search("iq2_xs", grids["iq2_xs"], wl["w"][r:r + 1],
                                                wl["hess"].numpy(), cand)
        assert np.array_equal(picks[r:r + 1].cpu().numpy(), want_p), r
        assert np.array_equal(pay[r:r + 1].cpu().numpy(), want_pay), r


def test_full_size_iq1s_64x256(dev, descs, grids, anchors):
    wl = synth.workload_iq1s_64x256()
    got = iq.iq_encode(descs["iq1_s"], wl["w"].to(dev)).cpu().numpy()
    want, _ = oracle.encode("iq1_s", grids["iq1_s"], anchors["iq1_s"], wl["w"])
    assert np.array_equal(got, want)
    dec = iq.iq_decode(descs["iq1_s"], torch.from_numpy(got).to(dev), torch.float32).cpu().numpy()
    assert np.array_equal(dec, oracle.decode("iq1_s", grids["iq1_s"], want))
