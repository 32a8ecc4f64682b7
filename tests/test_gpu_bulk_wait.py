"""The bounded wait on bulk copies into shared memory, which the choice search stages its H panels
with (include/iq_probe.h: iq_probe_bulk_wait).

A copy that completes is waited for and lands intact; a barrier no copy was issued for makes the
bounded wait run out, the kernel returns, and the context stays usable. Nothing here faults.
"""
import numpy as np
import pytest
import torch

import ggml_iq_codebook_b200 as iq

pytestmark = pytest.mark.gpu


def _weighted_sum(words: np.ndarray) -> int:
    w = words.astype(np.uint64)
    return int((w * (2 * np.arange(w.size, dtype=np.uint64) + 1)).sum() % (1 << 32))


@pytest.mark.parametrize("nbytes", [16, 1024, 4096])
def test_bulk_copy_completes_and_lands(nbytes):
    g = np.random.default_rng(nbytes)
    host = g.integers(0, 1 << 32, size=nbytes // 4, dtype=np.uint64).astype(np.uint32)
    src = torch.from_numpy(host.view(np.int32)).cuda()
    out = torch.zeros(2, dtype=torch.int32, device="cuda")
    iq.probe_bulk_wait(src, True, 200_000_000, out)
    got = out.cpu().numpy().view(np.uint32)
    assert got[0] == 1
    assert int(got[1]) == _weighted_sum(host)


def test_wait_without_copy_runs_out_and_returns():
    out = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    iq.probe_bulk_wait(None, False, 1_000_000, out)  # about half a millisecond of waiting
    torch.cuda.synchronize()
    assert out.cpu().tolist() == [0, 0]
    # the context is still usable: a completing copy right after
    src = torch.arange(64, dtype=torch.int32, device="cuda")
    iq.probe_bulk_wait(src, True, 200_000_000, out)
    assert int(out[0]) == 1


def test_bad_arguments_launch_nothing():
    lib = iq.load_library()
    out = torch.zeros(2, dtype=torch.int32, device="cuda")
    src = torch.zeros(1024, dtype=torch.int32, device="cuda")
    p = src.data_ptr()
    assert lib.iq_probe_bulk_wait(p + 4, 64, 1, 1000, out.data_ptr(), None) == 1  # src not 16-byte aligned
    assert lib.iq_probe_bulk_wait(p, 24, 1, 1000, out.data_ptr(), None) == 1      # not a multiple of 16
    assert lib.iq_probe_bulk_wait(p, 8192, 1, 1000, out.data_ptr(), None) == 1    # beyond the probe's 4 KiB
    assert lib.iq_probe_bulk_wait(p, 64, 1, 0, out.data_ptr(), None) == 1         # no wait bound
    assert lib.iq_probe_bulk_wait(p, 64, 1, 1000, None, None) == 1
