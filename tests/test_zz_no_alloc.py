"""The per-block calibration loop with the library's own scratch, for callers that cannot
allocate device memory at the call (needs a B200).

iq_gptq_blocks_static is iq_gptq_blocks without the workspace argument: code that runs inside
another framework's memory pool, or under a fixed device-memory budget, or where cudaMalloc's
implicit synchronisation is not acceptable, calls it instead and the library uses a fixed 10 MiB
device array of its own. This file calls it through the C ABI, twice in a row on different
weights (the array keeps the first call's contents, which must not leak into the second), and
requires the payloads, picks and compensated weights to equal what iq_gptq_blocks writes with a
caller-owned workspace, bit for bit (the tolerance every parity test here uses). It also checks
that a call needing more than the array holds is refused before anything runs.

The file is named to be collected last, so a run that stops at the first failure has run every
other test before it; it passes alone in a fresh process as well.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq
from ggml_iq_codebook_b200 import build, synth

pytestmark = pytest.mark.gpu

IQ_ESCRATCH = 10


def _inputs(rows, nblk, seed):
    w = synth.normal_bf16((rows, 256 * nblk), 0.02, seed)
    U = synth.inverse_hessian_factor(nblk, seed=seed + 100, cross_seed=seed + 200, cross_std=0.05)
    hess = torch.stack([synth.block_hessian(seed + 100 + b) for b in range(nblk)])
    return w, U, hess


def _static_call(lib, desc, w, hess, U, dev):
    rows, cols = w.shape
    nblk = cols // 256
    fmt = "iq2_xs"
    payload = torch.empty((rows, nblk, iq.BLOCK_BYTES[fmt]), dtype=torch.uint8, device=dev)
    picks = torch.empty((rows, nblk, iq.CHOICE_GROUPS[fmt]), dtype=torch.uint8, device=dev)
    w_work = torch.empty((rows, cols), dtype=torch.float32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    st = lib.iq_gptq_blocks_static(ctypes.byref(desc), w.data_ptr(), rows, cols, w.stride(0), hess.data_ptr(),
                                   U.data_ptr(), U.stride(0), payload.data_ptr(), picks.data_ptr(),
                                   w_work.data_ptr(), flags.data_ptr(),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.iq_status_string(st)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    return payload, picks, w_work


def test_static_scratch_equals_caller_workspace_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    lib = iq.load_library()
    dev = torch.device("cuda:0")
    grid = torch.from_numpy(synth.iq2xs_grid()).to(dev)
    desc = iq.make_desc("iq2_xs", grid)
    for rows, nblk, seed in ((200, 3, 501), (77, 2, 502)):
        w, U, hess = _inputs(rows, nblk, seed)
        wd, Ud, hd = w.to(dev), U.to(dev), hess.to(dev)
        got = _static_call(lib, desc, wd, hd, Ud, dev)
        want = iq.iq_gptq_blocks(desc, wd, hd, Ud)
        torch.cuda.synchronize()
        for g, wt in zip(got, want):
            assert np.array_equal(g.cpu().numpy().view(np.uint8), wt.cpu().numpy().view(np.uint8))

    # more rows than the 10 MiB array serves: refused before anything is enqueued
    rows = 5000
    assert iq.iq_gptq_workspace_bytes("iq2_xs", rows) > 10 << 20
    w = torch.zeros((rows, 256), dtype=torch.bfloat16, device=dev)
    hess = torch.zeros((1, 256, 256), dtype=torch.float32, device=dev)
    U = torch.zeros((256, 256), dtype=torch.float32, device=dev)
    out = torch.empty((rows, 1, 74), dtype=torch.uint8, device=dev)
    picks = torch.empty((rows, 1, 16), dtype=torch.uint8, device=dev)
    w_work = torch.empty((rows, 256), dtype=torch.float32, device=dev)
    st = lib.iq_gptq_blocks_static(ctypes.byref(desc), w.data_ptr(), rows, 256, 256, hess.data_ptr(), U.data_ptr(),
                                   256, out.data_ptr(), picks.data_ptr(), w_work.data_ptr(), None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == IQ_ESCRATCH
