"""Host-side checks of the C-ABI library (no GPU needed, no kernel launched)."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

import ggml_iq_codebook_b200 as iq
from ggml_iq_codebook_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return iq.load_library()


def _declared_functions(header=None):
    names = [header] if header else sorted(os.listdir(os.path.join(ROOT, "include")))
    out = set()
    for h in names:
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        out |= set(re.findall(r"\b(iq_[a-z0-9_]+)\s*\(", src))
    return sorted(out)


def test_header_declares_the_binding_symbols():
    assert set(_declared_functions("iq.h")) == set(iq.SYMBOLS)
    assert set(_declared_functions("iq_probe.h")) == set(iq.PROBE_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_format_tables(lib):
    assert lib.iq_block_bytes(1) == 50 and lib.iq_block_bytes(2) == 74 and lib.iq_block_bytes(3) == 56
    assert lib.iq_block_bytes(4) == 82 and lib.iq_block_bytes(5) == 0
    assert lib.iq_choice_groups(1) == 8 and lib.iq_choice_groups(2) == 16 and lib.iq_choice_groups(3) == 16
    assert lib.iq_num_choices(1) == 16 and lib.iq_num_choices(2) == 16 and lib.iq_num_choices(3) == 8
    assert lib.iq_num_choices(0) == 0
    for fmt, code in iq.IQ_FMT.items():
        assert lib.iq_block_bytes(code) == iq.BLOCK_BYTES[fmt]
        assert lib.iq_choice_groups(code) == iq.CHOICE_GROUPS[fmt]
        assert lib.iq_num_choices(code) == iq.CHOICES[fmt]
    assert b"sm_100a" in lib.iq_build_info()
    assert lib.iq_status_string(2).startswith(b"invalid shape")
    for st in range(12):
        assert lib.iq_status_string(st) != b"unknown status", st
    assert lib.iq_status_string(12) == b"unknown status"
    assert lib.iq_probe_fp32_ops_per_iter(0) == 8 and lib.iq_probe_fp32_ops_per_iter(3) == 16
    assert lib.iq_probe_fp32_ops_per_iter(4) == 0


def test_payload_bytes(lib):
    for fmt, code in iq.IQ_FMT.items():
        assert lib.iq_payload_bytes(code, 4096, 4096) == 4096 * 16 * iq.BLOCK_BYTES[fmt]
        assert lib.iq_payload_bytes(code, 0, 256) == 0 and lib.iq_payload_bytes(code, 3, 0) == 0
        assert lib.iq_payload_bytes(code, 2, 384) == 0 and lib.iq_payload_bytes(code, -1, 256) == 0
    assert lib.iq_payload_bytes(1, 256 * 1536, 4096) == 256 * 1536 * 16 * 50
    assert lib.iq_payload_bytes(7, 1, 256) == 0


def _desc(fmt=1, entries=2048, grid=0x1000, anchor=0.61):
    return iq.IQDesc(fmt, entries, grid, anchor)


def test_argument_errors_are_reported_before_any_launch(lib):
    E = lib.iq_encode
    d = _desc()
    W = 0x10000  # a fake, 16-byte aligned address: validation must fail before it is touched
    # bad descriptors
    assert E(None, W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(_desc(fmt=5)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(_desc(fmt=4, entries=512)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None,
             None) == 1
    assert E(ctypes.byref(_desc(fmt=3, entries=512)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None,
             None) == 1
    assert E(ctypes.byref(_desc(entries=512)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(_desc(anchor=float("nan"))), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(_desc(anchor=0.0)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(_desc(grid=0x1001)), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    # shapes: the [512, 384] case, empty tensors
    assert E(ctypes.byref(d), W, 0, 1, 512, 384, 384, 0, None, 0, None, None, 0, 0, W, None, None) == 2
    assert E(ctypes.byref(d), W, 0, 1, 0, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 2
    assert E(ctypes.byref(d), W, 0, 0, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 2
    # NULL buffers, strides, exclusive options
    assert E(ctypes.byref(d), None, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W, 0, 1, 4, 256, 128, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W + 2, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W, 0, 2, 4, 256, 256, 256, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W, 0, 1, 4, 256, 256, 0, None, 0, W, None, 0, 1, W, None, None) == 1
    assert E(ctypes.byref(d), W, 0, 1, 4, 256, 256, 0, None, 0, None, None, 0, 2, W, None, None) == 1
    # weight dtypes: an unknown kind; f16 rows must be a multiple of 8 elements (fp32: 4)
    assert E(ctypes.byref(d), W, 3, 1, 4, 256, 256, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W, 1, 1, 4, 256, 260, 0, None, 0, None, None, 0, 0, W, None, None) == 1
    # static scales: 2-byte aligned, stride >= 1
    assert E(ctypes.byref(d), W, 0, 1, 4, 256, 256, 0, None, 0, None, W + 1, 1, 0, W, None, None) == 1
    assert E(ctypes.byref(d), W, 0, 1, 4, 256, 256, 0, None, 0, None, W, 0, 0, W, None, None) == 1
    # decode / choice search / sqrt_diag
    assert lib.iq_decode(ctypes.byref(d), W, 0, 1, W, None) == 2
    assert lib.iq_decode(ctypes.byref(d), W, 4, 7, W, None) == 1
    assert lib.iq_decode(ctypes.byref(d), None, 4, 1, W, None) == 1
    assert lib.iq_choice_search(ctypes.byref(d), W, 0, 1, 256, W, 0, W, 1, 0, W, W, 1, None, None, None) == 2
    assert lib.iq_choice_search(ctypes.byref(d), W, 4, 2, 256, W, 0, W, 2, 0, W, W, 2, None, None, None) == 1
    assert lib.iq_choice_search(ctypes.byref(d), W, 6, 1, 256, W, 4, W, 1, 0, W, W, 1, None, None, None) == 2  # 4 !| 6
    # IQ1_M: any anchor (it is derived per block)
    m = _desc(fmt=3, anchor=float("nan"))
    assert E(ctypes.byref(m), W, 0, 1, 512, 384, 384, 0, None, 0, None, None, 0, 0, W, None, None) == 2
    assert lib.iq_choice_search(ctypes.byref(m), W, 4, 1, 256, W, 3, W, 1, 0, W, W, 1, None, None, None) == 2  # 3 !| 4
    s2 = _desc(fmt=4, entries=1024, anchor=0.9)
    assert lib.iq_choice_search(ctypes.byref(s2), W, 0, 1, 256, W, 0, W, 1, 0, W, W, 1, None, None, None) == 2
    # the 8-column choice search: IQ2_XS only; shapes and buffers as the 16-column one, no payload
    x2 = _desc(fmt=2, entries=512, anchor=0.9)
    G8 = lib.iq_choice_search_g8
    assert G8(ctypes.byref(d), W, 4, 1, 256, W, 0, W, 1, 0, W, None, None, None) == 4
    assert G8(ctypes.byref(x2), W, 0, 1, 256, W, 0, W, 1, 0, W, None, None, None) == 2
    assert G8(ctypes.byref(x2), W, 6, 1, 256, W, 4, W, 1, 0, W, None, None, None) == 2  # 4 !| 6
    assert G8(ctypes.byref(x2), W, 4, 1, 256, W, 0, W, 1, 0, None, None, None, None) == 1
    assert G8(ctypes.byref(x2), W, 4, 2, 256, W, 0, W, 2, 0, W, None, None, None) == 1  # ldw < 512
    assert G8(ctypes.byref(x2), W, 4, 1, 256, W, 0, W + 1, 1, 0, W, None, None, None) == 1
    assert G8(ctypes.byref(x2), W, 4, 1, 256, W, 0, W, 1, 3, W, None, None, None) == 1
    assert lib.iq_sqrt_diag(None, 1, W, None) == 1
    assert lib.iq_sqrt_diag(W, 0, W, None) == 2
