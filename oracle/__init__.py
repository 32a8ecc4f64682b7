"""CPU oracle for the GGML IQ encoder path -- TEST INFRASTRUCTURE ONLY.

A plain, slow C restatement (``iq_oracle.c``) of the IQ1_S / IQ1_M / IQ2_XS / IQ2_S encoder and
decoder, and the local-Hessian choice search (all four formats), with this thin ctypes wrapper.
It is the yardstick the CUDA library is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import it; the library
never does, and the two share no code.

Functions whose parity rests on invariants only (no value fixed by the pages or by a closed form)
are marked "parity unpinned" in their docstrings.
"""

from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "iq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FMT = {"iq1_s": 1, "iq2_xs": 2, "iq1_m": 3, "iq2_s": 4}
BLOCK_BYTES = {"iq1_s": 50, "iq2_xs": 74, "iq1_m": 56, "iq2_s": 82}
CHOICE_GROUPS = {"iq1_s": 8, "iq2_xs": 16, "iq1_m": 16, "iq2_s": 16}
CHOICES = {"iq1_s": 16, "iq2_xs": 16, "iq1_m": 8, "iq2_s": 16}
CS_IQ2XS_G8 = 5  # choice-search layout code: IQ2_XS candidates, 32 groups of 8 columns, ls 8..15
NUM_CHOICES = 16

FLAG_NONFINITE = 1
FLAG_IMPORTANCE = 2
FLAG_RANGE = 4
FLAG_CHOICE = 8
FLAG_GRID = 16

_lib = None


def build(force: bool = False) -> str:
    """Compile iq_oracle.c with gcc (-ffp-contract=off keeps a*b+c as two roundings)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O2", "-Wall", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def build_optimised() -> str:
    """The same source compiled with -O3 -march=native, still with -ffp-contract=off and without
    fast-math, so IEEE semantics (and every output bit) are the plain build's. It serves only the
    script that writes the stored full-size digests, where the plain build would take hours."""
    out = os.path.join(_HERE, "liboracle_O3.so")
    if not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-std=c11", "-O3", "-march=native", "-Wall", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-shared", "-fPIC", "-o", out + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(out + ".tmp", out)
    return out


def _load(path: str | None = None):
    global _lib
    if _lib is None or path is not None:
        lib = ctypes.CDLL(path or build())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.orc_encode.restype = ctypes.c_uint32
        lib.orc_encode.argtypes = [ctypes.c_int, P, ctypes.c_float, P, ctypes.c_int, i64, i64, P, P, ctypes.c_int,
                                   P, P]
        lib.orc_decode.restype = None
        lib.orc_decode.argtypes = [ctypes.c_int, P, P, i64, P]
        lib.orc_choice_search.restype = ctypes.c_uint32
        lib.orc_choice_search.argtypes = [ctypes.c_int, P, P, ctypes.c_int, i64, i64, i64, P, i64, P, P, P, P, P]
        lib.orc_gptq_blocks.restype = ctypes.c_uint32
        lib.orc_gptq_blocks.argtypes = [ctypes.c_int, P, ctypes.c_float, P, i64, i64, P, P, P, P, P]
        lib.orc_sqrt_diag.restype = None
        lib.orc_sqrt_diag.argtypes = [P, i64, P]
        lib.orc_f32_to_f16.restype = ctypes.c_uint16
        lib.orc_f32_to_f16.argtypes = [ctypes.c_float]
        lib.orc_f16_to_f32.restype = ctypes.c_float
        lib.orc_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.orc_f32_to_bf16_array.restype = None
        lib.orc_f32_to_bf16_array.argtypes = [P, i64, P]
        lib.orc_set_threads.argtypes = [ctypes.c_int]
        lib.orc_get_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


@contextlib.contextmanager
def library(path: str):
    """Temporarily run every oracle call through another build of iq_oracle.c (used by the
    mutation test, which plants mistakes in a copy of the source and expects the pins to fail)."""
    global _lib
    saved = _lib
    _load(path)
    try:
        yield
    finally:
        _lib = saved


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(w) -> np.ndarray:
    """Accept a torch bf16 tensor or a uint16 array of bf16 bit patterns."""
    if hasattr(w, "view") and hasattr(w, "dtype") and str(w.dtype) == "torch.bfloat16":
        import torch
        return np.ascontiguousarray(w.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    return np.ascontiguousarray(np.asarray(w, dtype=np.uint16))


IN_BF16, IN_F16, IN_F32 = 0, 1, 2


def _weights(w):
    """(contiguous array, element kind) for a torch bf16/f16/f32 tensor, a numpy float32/float16
    array, or a uint16 array of bf16 bit patterns."""
    if hasattr(w, "dtype") and str(w.dtype).startswith("torch."):
        import torch
        t = w.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return np.ascontiguousarray(t.view(torch.int16).numpy().view(np.uint16)), IN_BF16
        if t.dtype == torch.float16:
            return np.ascontiguousarray(t.view(torch.int16).numpy().view(np.uint16)), IN_F16
        if t.dtype == torch.float32:
            return np.ascontiguousarray(t.numpy()), IN_F32
        raise TypeError(f"unsupported weight dtype {t.dtype}")
    a = np.asarray(w)
    if a.dtype == np.float32:
        return np.ascontiguousarray(a), IN_F32
    if a.dtype == np.float16:
        return np.ascontiguousarray(a.view(np.uint16)), IN_F16
    return np.ascontiguousarray(a.astype(np.uint16)), IN_BF16


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def threads() -> int:
    return int(_load().orc_get_threads())


def f32_to_f16_bits(v: float) -> int:
    return int(_load().orc_f32_to_f16(float(v)))


def f16_bits_to_f32(h: int) -> float:
    return float(_load().orc_f16_to_f32(int(h)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().orc_f32_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def encode(fmt: str, grid: np.ndarray, anchor: float, w, importance=None, choices=None,
           every_choice: bool = False, scales=None):
    """Encode a [rows, cols] weight (bf16, f16 or f32; see _weights). Returns (payload uint8, flags).

    payload: [rows, cols/256, B], or [C, rows, cols/256, B] with every_choice (C = 16; 8 for iq1_m).
    anchor is ignored for iq1_m, whose anchor follows each block's peak-to-RMS.
    scales: optional [rows, cols/256] fp16 values (or their uint16 bits): encode under these d.
    """
    lib = _load()
    wb, kind = _weights(w)
    rows, cols = wb.shape
    if cols % 256:
        raise ValueError("cols must be a multiple of 256")
    nblk = cols // 256
    B = BLOCK_BYTES[fmt]
    grid = np.ascontiguousarray(grid, dtype=np.int8)
    imp = None if importance is None else np.ascontiguousarray(np.asarray(importance, dtype=np.float32))
    ch = None if choices is None else np.ascontiguousarray(np.asarray(choices, dtype=np.uint8))
    sc = None
    if scales is not None:
        sc = np.asarray(scales)
        sc = np.ascontiguousarray(sc.view(np.uint16) if sc.dtype == np.float16 else sc.astype(np.uint16))
    shape = (CHOICES[fmt], rows, nblk, B) if every_choice else (rows, nblk, B)
    out = np.zeros(shape, dtype=np.uint8)
    flags = lib.orc_encode(FMT[fmt], _ptr(grid), float(anchor), _ptr(wb), kind, rows, cols, _ptr(imp),
                           _ptr(ch), int(bool(every_choice)), _ptr(sc), _ptr(out))
    return out, int(flags)


def decode(fmt: str, grid: np.ndarray, payload: np.ndarray) -> np.ndarray:
    """Decode payload [..., B] to fp32 [..., 256] (exact)."""
    B = BLOCK_BYTES[fmt]
    p = np.ascontiguousarray(payload, dtype=np.uint8)
    nblocks = p.size // B
    out = np.empty(p.shape[:-1] + (256,), dtype=np.float32)
    _load().orc_decode(FMT[fmt], _ptr(np.ascontiguousarray(grid, dtype=np.int8)), _ptr(p), nblocks, _ptr(out))
    return out


def choice_search(fmt: str, grid: np.ndarray, w, hess: np.ndarray, cand: np.ndarray, trace=False,
                  objective=False, return_flags=False):
    """Local-Hessian choice search over every 256-column block of w.

    w: [rows, cols] (bf16, or fp32 values), or [experts, rows, cols] with hess [experts, nblk, 256, 256] (each expert's
    rows use its own Hessian blocks); hess: [nblk, 256, 256] fp32 otherwise;
    cand: [C, (experts,) rows, nblk, B] every-choice payloads (C = 16; 8 for iq1_m).
    Returns (picks [(experts,) rows, nblk, G], payload [(experts,) rows, nblk, B]) and, with
    trace, the picks after step 2 and after each sweep [(experts,) rows, nblk, 3, G]; with objective
    (after the picks and payload, or the trace), each row-block's final Delta^T H Delta
    [(experts,) rows, nblk] fp32; with return_flags (last), the findings word (FLAG_NONFINITE for a
    non-finite weight or Hessian entry, FLAG_GRID for a grid value outside the alphabet). A
    row-block with a finding gets picks 0, the all-zero payload and a NaN objective.
    Parity of the sweeps is pinned by the fp64 direct-objective replay in the tests.
    """
    wb, kind = _weights(w)
    if kind == IN_F16:
        raise TypeError("the choice search takes bf16 or fp32 weights")
    lead = wb.shape[:-1]
    cols = wb.shape[-1]
    wb = wb.reshape(-1, cols)
    rows = wb.shape[0]
    nexp = wb.shape[0] // lead[-1] if len(lead) == 2 else 1
    nblk = cols // 256
    G, B = CHOICE_GROUPS[fmt], BLOCK_BYTES[fmt]
    hess = np.ascontiguousarray(hess, dtype=np.float32).reshape(nexp, nblk, 256, 256)
    cand = np.ascontiguousarray(cand, dtype=np.uint8).reshape(CHOICES[fmt], rows, nblk, B)
    picks = np.zeros((rows, nblk, G), dtype=np.uint8)
    payload = np.zeros((rows, nblk, B), dtype=np.uint8)
    tr = np.zeros((rows, nblk, 3, G), dtype=np.uint8) if trace else None
    obj = np.zeros((rows, nblk), dtype=np.float32) if objective else None
    flags = _load().orc_choice_search(FMT[fmt], _ptr(np.ascontiguousarray(grid, dtype=np.int8)), _ptr(wb), kind,
                                      rows, nblk, cols, _ptr(hess), rows // nexp, _ptr(cand), _ptr(picks),
                                      _ptr(payload), _ptr(tr), _ptr(obj))
    out = [picks.reshape(lead + (nblk, G)), payload.reshape(lead + (nblk, B))]
    if trace:
        out.append(tr.reshape(lead + (nblk, 3, G)))
    if objective:
        out.append(obj.reshape(lead + (nblk,)))
    if return_flags:
        out.append(int(flags))
    return tuple(out)


def choice_search_g8(grid: np.ndarray, w, hess: np.ndarray, cand: np.ndarray, trace=False,
                     objective=False, return_flags=False):
    """The local-Hessian choice search with eight candidates per 8-weight group: 32 groups of 8
    columns per block, each choosing among the IQ2_XS every-choice decodes for ls = 8..15.

    w and hess as in choice_search; cand: the 16-choice IQ2_XS every-choice encode
    [16, (experts,) rows, nblk, 74], of which choices 8..15 are read. Returns (picks,) with picks
    [(experts,) rows, nblk, 32] holding the chosen ls (8..15); with trace, also the picks after
    step 2 and after each sweep [(experts,) rows, nblk, 3, 32]; with objective (last), each
    row-block's final Delta^T H Delta; with return_flags (last), the findings word, as in
    choice_search (a row-block with a finding gets picks 8). No payload layout stores a scale per
    8 weights, so none is assembled.
    """
    wb, kind = _weights(w)
    if kind == IN_F16:
        raise TypeError("the choice search takes bf16 or fp32 weights")
    lead = wb.shape[:-1]
    cols = wb.shape[-1]
    wb = wb.reshape(-1, cols)
    rows = wb.shape[0]
    nexp = wb.shape[0] // lead[-1] if len(lead) == 2 else 1
    nblk = cols // 256
    hess = np.ascontiguousarray(hess, dtype=np.float32).reshape(nexp, nblk, 256, 256)
    cand = np.ascontiguousarray(cand, dtype=np.uint8).reshape(16, rows, nblk, 74)
    picks = np.zeros((rows, nblk, 32), dtype=np.uint8)
    tr = np.zeros((rows, nblk, 3, 32), dtype=np.uint8) if trace else None
    obj = np.zeros((rows, nblk), dtype=np.float32) if objective else None
    flags = _load().orc_choice_search(CS_IQ2XS_G8, _ptr(np.ascontiguousarray(grid, dtype=np.int8)), _ptr(wb),
                                      kind, rows, nblk, cols, _ptr(hess), rows // nexp, _ptr(cand), _ptr(picks),
                                      None, _ptr(tr), _ptr(obj))
    out = [picks.reshape(lead + (nblk, 32))]
    if trace:
        out.append(tr.reshape(lead + (nblk, 3, 32)))
    if objective:
        out.append(obj.reshape(lead + (nblk,)))
    if return_flags:
        out.append(int(flags))
    return tuple(out)


def gptq_blocks(fmt: str, grid: np.ndarray, anchor: float, w, hess: np.ndarray, U: np.ndarray):
    """The per-block calibration loop over one bf16 weight [rows, cols]: for each 256-column block
    in order, the every-choice encode under sqrt(diag H_b), the local-Hessian choice search under
    H_b, then GPTQ's propagation of the block's error E to the later columns through U (the upper
    Cholesky factor of the inverse Hessian, [cols, cols]; hess: [cols/256, 256, 256]).
    Returns (payload [rows, nblk, B], picks [rows, nblk, G], w_work [rows, cols] fp32: the weights
    each block was quantised from, flags)."""
    wb = _bf16_bits(w)
    rows, cols = wb.shape
    nblk = cols // 256
    B, G = BLOCK_BYTES[fmt], CHOICE_GROUPS[fmt]
    hess = np.ascontiguousarray(hess, dtype=np.float32).reshape(nblk, 256, 256)
    U = np.ascontiguousarray(U, dtype=np.float32).reshape(cols, cols)
    payload = np.zeros((rows, nblk, B), dtype=np.uint8)
    picks = np.zeros((rows, nblk, G), dtype=np.uint8)
    w_work = np.zeros((rows, cols), dtype=np.float32)
    flags = _load().orc_gptq_blocks(FMT[fmt], _ptr(np.ascontiguousarray(grid, dtype=np.int8)), float(anchor),
                                    _ptr(wb), rows, cols, _ptr(hess), _ptr(U), _ptr(payload), _ptr(picks),
                                    _ptr(w_work))
    return payload, picks, w_work, int(flags)


def sqrt_diag(hess: np.ndarray) -> np.ndarray:
    """sqrt of the diagonal of each [256, 256] block: the candidates' search importance."""
    h = np.ascontiguousarray(hess, dtype=np.float32).reshape(-1, 256, 256)
    out = np.empty((h.shape[0] * 256,), dtype=np.float32)
    _load().orc_sqrt_diag(_ptr(h), h.shape[0], _ptr(out))
    return out
