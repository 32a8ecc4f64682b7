"""Python binding of libiq_b200 (the B200 GGML IQ encoder library).

Thin ctypes marshalling over the C ABI in include/iq.h: torch tensors supply device memory and
the current CUDA stream, every computation runs in the library's kernels. There is no CPU path:
if the shared library is missing or the device is not an sm_100 part, calls raise.

Functions keep the C names: iq_encode, iq_decode, iq_choice_search, iq_choice_search_g8,
iq_sqrt_diag.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libiq_b200.so")

IQ_FMT = {"iq1_s": 1, "iq2_xs": 2, "iq1_m": 3, "iq2_s": 4}
BLOCK_BYTES = {"iq1_s": 50, "iq2_xs": 74, "iq1_m": 56, "iq2_s": 82}
CHOICE_GROUPS = {"iq1_s": 8, "iq2_xs": 16, "iq1_m": 16, "iq2_s": 16}
GRID_ENTRIES = {"iq1_s": 2048, "iq2_xs": 512, "iq1_m": 2048, "iq2_s": 1024}
CHOICES = {"iq1_s": 16, "iq2_xs": 16, "iq1_m": 8, "iq2_s": 16}
NUM_CHOICES = 16
# d = fp16(fp32(amax / qmax) * anchor): IQ1_S's 0.61 is the pages' constant; IQ2_XS's was fixed
# once by a seeded sweep on non-evaluation data (the pages name a clamp but give no numbers).
# IQ1_M ignores the descriptor's anchor: it follows each block's peak-to-RMS.
DEFAULT_ANCHOR = {"iq1_s": 0.61, "iq2_xs": 0.9, "iq1_m": 1.0, "iq2_s": 0.9}

IQ_OUT_F32, IQ_OUT_BF16 = 0, 1
IQ_IN = {torch.bfloat16: 0, torch.float16: 1, torch.float32: 2}
FLAG_NONFINITE, FLAG_IMPORTANCE, FLAG_RANGE, FLAG_CHOICE, FLAG_GRID, FLAG_TIMEOUT = 1, 2, 4, 8, 16, 32

SYMBOLS = ("iq_block_bytes", "iq_payload_bytes", "iq_choice_groups", "iq_num_choices", "iq_encode", "iq_decode",
           "iq_choice_search", "iq_choice_search_g8", "iq_gptq_workspace_bytes", "iq_gptq_blocks",
           "iq_gptq_blocks_static", "iq_sqrt_diag",
           "iq_status_string", "iq_build_info")
PROBE_SYMBOLS = ("iq_probe_fp32", "iq_probe_fp32_ops_per_iter", "iq_probe_bulk_wait")  # include/iq_probe.h


class IQError(RuntimeError):
    """A non-OK status from the library, or a device-side finding in the flags word."""


class IQDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("grid_entries", ctypes.c_int32),
                ("grid", ctypes.c_void_p), ("anchor", ctypes.c_float)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libiq_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise IQError(f"{path} is missing: build it with ggml_iq_codebook_b200.build.build()")
    lib = ctypes.CDLL(path)
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    lib.iq_block_bytes.restype = ctypes.c_size_t
    lib.iq_block_bytes.argtypes = [i32]
    lib.iq_payload_bytes.restype = ctypes.c_size_t
    lib.iq_payload_bytes.argtypes = [i32, i64, i64]
    lib.iq_choice_groups.restype = i32
    lib.iq_choice_groups.argtypes = [i32]
    lib.iq_num_choices.restype = i32
    lib.iq_num_choices.argtypes = [i32]
    lib.iq_encode.restype = ctypes.c_int
    lib.iq_encode.argtypes = [ctypes.POINTER(IQDesc), P, i32, i64, i64, i64, i64, i64, P, i64, P, P, i64, i32, P, P,
                              P]
    lib.iq_decode.restype = ctypes.c_int
    lib.iq_decode.argtypes = [ctypes.POINTER(IQDesc), P, i64, i32, P, P]
    lib.iq_choice_search.restype = ctypes.c_int
    lib.iq_choice_search.argtypes = [ctypes.POINTER(IQDesc), P, i64, i64, i64, P, i64, P, i64, i64, P, P, i64, P, P,
                                     P]
    lib.iq_choice_search_g8.restype = ctypes.c_int
    lib.iq_choice_search_g8.argtypes = [ctypes.POINTER(IQDesc), P, i64, i64, i64, P, i64, P, i64, i64, P, P, P, P]
    lib.iq_gptq_workspace_bytes.restype = ctypes.c_size_t
    lib.iq_gptq_workspace_bytes.argtypes = [i32, i64]
    lib.iq_gptq_blocks.restype = ctypes.c_int
    lib.iq_gptq_blocks.argtypes = [ctypes.POINTER(IQDesc), P, i64, i64, i64, P, P, i64, P, ctypes.c_size_t, P, P, P,
                                   P, P]
    lib.iq_gptq_blocks_static.restype = ctypes.c_int
    lib.iq_gptq_blocks_static.argtypes = [ctypes.POINTER(IQDesc), P, i64, i64, i64, P, P, i64, P, P, P, P, P]
    lib.iq_sqrt_diag.restype = ctypes.c_int
    lib.iq_sqrt_diag.argtypes = [P, i64, P, P]
    lib.iq_status_string.restype = ctypes.c_char_p
    lib.iq_status_string.argtypes = [ctypes.c_int]
    lib.iq_build_info.restype = ctypes.c_char_p
    lib.iq_probe_fp32.restype = i32
    lib.iq_probe_fp32.argtypes = [i32, i64, i64, P, P]
    lib.iq_probe_fp32_ops_per_iter.restype = i64
    lib.iq_probe_fp32_ops_per_iter.argtypes = [i32]
    lib.iq_probe_bulk_wait.restype = i32
    lib.iq_probe_bulk_wait.argtypes = [P, i64, i32, i64, P, P]
    _lib = lib
    return lib


def _check(status: int) -> None:
    if status != 0:
        raise IQError(f"libiq_b200: {load_library().iq_status_string(status).decode()} (status {status})")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise IQError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise IQError(f"{name} must be {dtype}, got {t.dtype}")


def make_desc(fmt: str, grid: torch.Tensor, anchor: float | None = None) -> IQDesc:
    """Descriptor for a device grid ([2048, 8] or [512, 8] int8)."""
    _need(grid, torch.int8, "grid")
    if tuple(grid.shape) != (GRID_ENTRIES[fmt], 8) or not grid.is_contiguous():
        raise IQError(f"grid must be a contiguous [{GRID_ENTRIES[fmt]}, 8] int8 tensor")
    d = IQDesc(IQ_FMT[fmt], GRID_ENTRIES[fmt], grid.data_ptr(),
               DEFAULT_ANCHOR[fmt] if anchor is None else float(anchor))
    d._grid_ref = grid  # keep the device grid alive with the descriptor
    return d


def _fmt_of(desc: IQDesc) -> str:
    return {1: "iq1_s", 2: "iq2_xs", 3: "iq1_m", 4: "iq2_s"}[desc.fmt]


def iq_encode(desc: IQDesc, w: torch.Tensor, importance: torch.Tensor | None = None,
              choices: torch.Tensor | None = None, every_choice: bool = False,
              out: torch.Tensor | None = None, flags: torch.Tensor | None = None, stream=None,
              raise_on_flags: bool = True, scales: torch.Tensor | None = None) -> torch.Tensor:
    """Encode weights [rows, cols] or [batch, rows, cols] (bf16, f16 or f32; last dim contiguous).

    importance: fp32 [cols] or [batch, cols]; choices: uint8 [..., rows, cols/256, G].
    scales: static block scales, either fp16 [..., rows, cols/256] (contiguous) or, except for
    IQ1_M, an existing payload uint8 [..., rows, cols/256, B] whose d fields are read in place.
    Returns the payload uint8 [(C,) (batch,) rows, cols/256, B], C = CHOICES[fmt]. With
    raise_on_flags (default) the call synchronises and raises on a device-side finding; pass a flags tensor and
    raise_on_flags=False to stay asynchronous. flags=False passes no findings word: the library
    then synchronises itself and the call raises IQError with the finding's status (invalid
    blocks are written as zero payloads either way).
    """
    lib = load_library()
    fmt = _fmt_of(desc)
    if not isinstance(w, torch.Tensor) or not w.is_cuda or w.dtype not in IQ_IN:
        raise IQError("w must be a CUDA tensor of bfloat16, float16 or float32")
    batched = w.dim() == 3
    if w.dim() not in (2, 3) or w.stride(-1) != 1:
        raise IQError("w must be [rows, cols] or [batch, rows, cols] with a contiguous last dim")
    batch = w.shape[0] if batched else 1
    rows, cols = w.shape[-2], w.shape[-1]
    ldw = w.stride(-2)
    wbs = w.stride(0) if batched else 0
    imp_ptr, imp_bs = None, 0
    if importance is not None:
        _need(importance, torch.float32, "importance")
        if importance.stride(-1) != 1 or importance.shape[-1] != cols:
            raise IQError("importance must be [cols] or [batch, cols] with a contiguous last dim")
        imp_ptr = importance.data_ptr()
        imp_bs = importance.stride(0) if importance.dim() == 2 else 0
    ch_ptr = None
    if choices is not None:
        _need(choices, torch.uint8, "choices")
        want = (batch, rows, cols // 256, CHOICE_GROUPS[fmt])
        if choices.numel() != batch * rows * (cols // 256) * CHOICE_GROUPS[fmt] or not choices.is_contiguous():
            raise IQError(f"choices must be a contiguous uint8 tensor of {want} elements")
        ch_ptr = choices.data_ptr()
    sc_ptr, sc_stride = None, 0
    nb = batch * rows * (cols // 256)
    if scales is not None:
        if scales.device != w.device or not scales.is_contiguous():
            raise IQError("scales must be a contiguous tensor on the weight's device")
        if scales.dtype == torch.float16 and scales.numel() == nb:
            sc_stride = 1
        elif fmt != "iq1_m" and scales.dtype == torch.uint8 and scales.shape[-1] == BLOCK_BYTES[fmt] and \
                scales.numel() == nb * BLOCK_BYTES[fmt]:
            sc_stride = BLOCK_BYTES[fmt] // 2
        else:
            raise IQError(f"scales must be fp16 with {nb} elements or a payload of {nb} blocks")
        sc_ptr = scales.data_ptr()
    shape = ((CHOICES[fmt],) if every_choice else ()) + ((batch,) if batched else ()) + \
        (rows, cols // 256, BLOCK_BYTES[fmt])
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=w.device)
    elif tuple(out.shape) != shape or out.dtype != torch.uint8 or not out.is_contiguous():
        raise IQError(f"out must be a contiguous uint8 tensor of shape {shape}")
    if flags is None:
        flags = torch.empty(1, dtype=torch.int32, device=w.device)
    flags_ptr = None if flags is False else flags.data_ptr()
    _check(lib.iq_encode(ctypes.byref(desc), w.data_ptr(), IQ_IN[w.dtype], batch, rows, cols, ldw, wbs, imp_ptr, imp_bs,
                         ch_ptr, sc_ptr, sc_stride, int(bool(every_choice)), out.data_ptr(), flags_ptr,
                         _stream(stream)))
    if raise_on_flags and flags is not False:
        raise_for_flags(flags)
    return out


def raise_for_flags(flags: torch.Tensor) -> None:
    """Synchronise on the flags word and raise if the kernels reported a finding."""
    f = int(flags.item())
    if f:
        names = [n for n, b in (("non-finite weight", FLAG_NONFINITE), ("bad importance", FLAG_IMPORTANCE),
                                ("d overflows fp16", FLAG_RANGE), ("choice out of range", FLAG_CHOICE),
                                ("grid value outside the alphabet", FLAG_GRID),
                                ("a bounded copy wait ran out", FLAG_TIMEOUT)) if f & b]
        err = IQError("device-side finding: " + ", ".join(names))
        err.flags = f
        raise err


def iq_decode(desc: IQDesc, payload: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16,
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode payload [..., B] to [..., 256] values (fp32 exact, or bf16)."""
    lib = load_library()
    fmt = _fmt_of(desc)
    _need(payload, torch.uint8, "payload")
    B = BLOCK_BYTES[fmt]
    if payload.shape[-1] != B or not payload.is_contiguous():
        raise IQError(f"payload must be contiguous with last dim {B}")
    nblocks = payload.numel() // B
    if out_dtype not in (torch.float32, torch.bfloat16):
        raise IQError("out_dtype must be float32 or bfloat16")
    shape = tuple(payload.shape[:-1]) + (256,)
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=payload.device)
    elif out.dtype != out_dtype or out.numel() != nblocks * 256 or not out.is_contiguous():
        raise IQError("out has the wrong dtype or size")
    _check(lib.iq_decode(ctypes.byref(desc), payload.data_ptr(), nblocks,
                         IQ_OUT_BF16 if out_dtype == torch.bfloat16 else IQ_OUT_F32, out.data_ptr(),
                         _stream(stream)))
    return out


def _blocks_ld(t: torch.Tensor, lead: tuple, nblk: int, B: int, name: str) -> int:
    """Row stride in blocks of a [..., (experts,) rows, nblk, B] uint8 view whose blocks are
    contiguous and whose rows (across experts too) are evenly spaced; raises otherwise."""
    tail = lead + (nblk, B)
    if t.dtype != torch.uint8 or tuple(t.shape[-len(tail):]) != tail:
        raise IQError(f"{name} must be uint8 [..., {', '.join(map(str, tail))}]")
    if t.stride(-1) != 1 or t.stride(-2) != B or t.stride(-3) % B != 0 or t.stride(-3) < nblk * B:
        raise IQError(f"{name}: each block must be contiguous and each row's blocks adjacent")
    if len(lead) == 2 and lead[0] > 1 and t.stride(-4) != lead[1] * t.stride(-3):
        raise IQError(f"{name}: the experts' rows must be evenly spaced")
    return t.stride(-3) // B


def _choice_args(desc: IQDesc, w: torch.Tensor, hess: torch.Tensor, cand: torch.Tensor, nchoice: int):
    """Checks shared by both choice searches: (fmt, lead, rows, rows per Hessian set, nblk, cand_ld)."""
    fmt = _fmt_of(desc)
    _need(w, torch.bfloat16, "w")
    _need(hess, torch.float32, "hess")
    _need(cand, torch.uint8, "cand")
    if w.dim() not in (2, 3) or w.stride(-1) != 1:
        raise IQError("w must be [rows, cols] or [experts, rows, cols] with a contiguous last dim")
    lead, cols = tuple(w.shape[:-1]), w.shape[-1]
    if cols == 0 or cols % 256:
        raise IQError(f"w must have a positive multiple of 256 columns, got {cols}")
    nexp, rows_e = (lead[0], lead[1]) if w.dim() == 3 else (1, lead[0])
    if w.dim() == 3 and nexp > 1 and w.stride(0) != rows_e * w.stride(1):
        raise IQError("the experts of w must be evenly spaced in the row dimension")
    nblk = cols // 256
    B = BLOCK_BYTES[fmt]
    if not hess.is_contiguous() or hess.numel() != nexp * nblk * 256 * 256:
        raise IQError("hess must be contiguous [(experts,) cols/256, 256, 256]")
    if cand.dim() != len(lead) + 3 or cand.shape[0] != nchoice:
        raise IQError(f"cand must be [{nchoice}, (experts,) rows, cols/256, {B}]")
    return fmt, lead, nexp * rows_e, rows_e, nblk, _blocks_ld(cand, lead, nblk, B, "cand")


def _objective_ok(objective, lead, nblk):
    if objective is not None and (objective.dtype != torch.float32 or tuple(objective.shape) != lead + (nblk,)
                                  or not objective.is_contiguous() or not objective.is_cuda):
        raise IQError(f"objective must be a contiguous float32 CUDA tensor of shape {lead + (nblk,)}")


def iq_choice_search(desc: IQDesc, w: torch.Tensor, hess: torch.Tensor, cand: torch.Tensor,
                     picks: torch.Tensor | None = None, payload: torch.Tensor | None = None,
                     flags: torch.Tensor | None = None, stream=None, objective: torch.Tensor | None = None):
    """Local-Hessian choice search over all 256-column blocks of w.

    w: bf16 [rows, cols] with hess fp32 [cols/256, 256, 256], or a stack of experts
    [experts, rows, cols] with hess [experts, cols/256, 256, 256] (each expert's rows use its own
    Hessian blocks; the experts must be evenly spaced in the row dimension).
    cand: uint8 [C, (experts,) rows, cols/256, B], the every-choice payloads (C = CHOICES[fmt]).
    w, cand and payload may be views (say one 256-column block of a wider weight and its slices):
    rows need only be evenly spaced, each block contiguous.
    objective: optional contiguous fp32 [(experts,) rows, cols/256], filled with each row-block's
    final Delta^T H Delta.
    Returns (picks uint8 [(experts,) rows, cols/256, G] contiguous, payload uint8
    [(experts,) rows, cols/256, B]).
    """
    lib = load_library()
    fmt, lead, rows, rows_e, nblk, cand_ld = _choice_args(desc, w, hess, cand, CHOICES[_fmt_of(desc)])
    B, G = BLOCK_BYTES[fmt], CHOICE_GROUPS[fmt]
    if picks is None:
        picks = torch.empty(lead + (nblk, G), dtype=torch.uint8, device=w.device)
    elif picks.dtype != torch.uint8 or tuple(picks.shape) != lead + (nblk, G) or not picks.is_contiguous():
        raise IQError(f"picks must be a contiguous uint8 tensor of shape {lead + (nblk, G)}")
    if payload is None:
        payload = torch.empty(lead + (nblk, B), dtype=torch.uint8, device=w.device)
    payload_ld = _blocks_ld(payload, lead, nblk, B, "payload")
    _objective_ok(objective, lead, nblk)
    _check(lib.iq_choice_search(ctypes.byref(desc), w.data_ptr(), rows, nblk, w.stride(-2), hess.data_ptr(),
                                rows_e, cand.data_ptr(), cand_ld, cand.stride(0), picks.data_ptr(),
                                payload.data_ptr(), payload_ld, None if objective is None else objective.data_ptr(),
                                None if flags is None else flags.data_ptr(), _stream(stream)))
    return picks, payload


def iq_choice_search_g8(desc: IQDesc, w: torch.Tensor, hess: torch.Tensor, cand: torch.Tensor,
                        picks: torch.Tensor | None = None, flags: torch.Tensor | None = None, stream=None,
                        objective: torch.Tensor | None = None) -> torch.Tensor:
    """The choice search with eight candidates per 8-weight group (IQ2_XS only): 32 groups of 8
    columns per block, each choosing among the every-choice decodes for ls = 8..15.

    w, hess, objective as in iq_choice_search; cand: uint8 [16, (experts,) rows, cols/256, 74],
    the IQ2_XS every-choice payloads (choices 8..15 are read). Returns picks uint8
    [(experts,) rows, cols/256, 32] holding the chosen ls (8..15); no payload is written.
    """
    lib = load_library()
    if _fmt_of(desc) != "iq2_xs":
        raise IQError("iq_choice_search_g8 takes IQ2_XS candidates")
    fmt, lead, rows, rows_e, nblk, cand_ld = _choice_args(desc, w, hess, cand, CHOICES["iq2_xs"])
    if picks is None:
        picks = torch.empty(lead + (nblk, 32), dtype=torch.uint8, device=w.device)
    elif picks.dtype != torch.uint8 or tuple(picks.shape) != lead + (nblk, 32) or not picks.is_contiguous():
        raise IQError(f"picks must be a contiguous uint8 tensor of shape {lead + (nblk, 32)}")
    _objective_ok(objective, lead, nblk)
    _check(lib.iq_choice_search_g8(ctypes.byref(desc), w.data_ptr(), rows, nblk, w.stride(-2), hess.data_ptr(),
                                   rows_e, cand.data_ptr(), cand_ld, cand.stride(0), picks.data_ptr(),
                                   None if objective is None else objective.data_ptr(),
                                   None if flags is None else flags.data_ptr(), _stream(stream)))
    return picks


def iq_gptq_workspace_bytes(fmt: str, rows: int) -> int:
    return int(load_library().iq_gptq_workspace_bytes(IQ_FMT[fmt], rows))


def iq_gptq_blocks(desc: IQDesc, w: torch.Tensor, hess: torch.Tensor, U: torch.Tensor,
                   workspace: torch.Tensor | None = None, payload: torch.Tensor | None = None,
                   picks: torch.Tensor | None = None, w_work: torch.Tensor | None = None,
                   flags: torch.Tensor | None = None, stream=None):
    """The per-block calibration loop over one bf16 weight [rows, cols] in one call: for each
    256-column block in order, the every-choice encode under sqrt(diag H_b), the local-Hessian
    choice search under H_b, and GPTQ's propagation of the block's error to the later columns
    through U (fp32 [cols, cols] upper-triangular factor of the inverse Hessian; hess fp32
    [cols/256, 256, 256]). workspace: uint8 CUDA tensor of iq_gptq_workspace_bytes(fmt, rows)
    bytes (allocated here if omitted). Returns (payload uint8 [rows, cols/256, B], picks uint8
    [rows, cols/256, G], w_work fp32 [rows, cols]: the weights each block was quantised from)."""
    lib = load_library()
    fmt = _fmt_of(desc)
    _need(w, torch.bfloat16, "w")
    _need(hess, torch.float32, "hess")
    _need(U, torch.float32, "U")
    if w.dim() != 2 or w.stride(-1) != 1:
        raise IQError("w must be [rows, cols] with a contiguous last dim")
    rows, cols = w.shape
    if cols == 0 or cols % 256:
        raise IQError(f"w must have a positive multiple of 256 columns, got {cols}")
    nblk = cols // 256
    if not hess.is_contiguous() or hess.numel() != nblk * 256 * 256:
        raise IQError("hess must be contiguous [cols/256, 256, 256]")
    if U.dim() != 2 or U.shape[0] != cols or U.shape[1] < cols or U.stride(-1) != 1:
        raise IQError("U must be [cols, >= cols] with a contiguous last dim")
    B, G = BLOCK_BYTES[fmt], CHOICE_GROUPS[fmt]
    need = iq_gptq_workspace_bytes(fmt, rows)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=w.device)
    elif workspace.dtype != torch.uint8 or workspace.numel() < need or not workspace.is_contiguous():
        raise IQError(f"workspace must be a contiguous uint8 tensor of at least {need} bytes")
    if payload is None:
        payload = torch.empty((rows, nblk, B), dtype=torch.uint8, device=w.device)
    if picks is None:
        picks = torch.empty((rows, nblk, G), dtype=torch.uint8, device=w.device)
    if w_work is None:
        w_work = torch.empty((rows, cols), dtype=torch.float32, device=w.device)
    for t, shape, dt, name in ((payload, (rows, nblk, B), torch.uint8, "payload"), (picks, (rows, nblk, G), torch.uint8,
                               "picks"), (w_work, (rows, cols), torch.float32, "w_work")):
        if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous():
            raise IQError(f"{name} must be a contiguous {dt} tensor of shape {shape}")
    _check(lib.iq_gptq_blocks(ctypes.byref(desc), w.data_ptr(), rows, cols, w.stride(0), hess.data_ptr(),
                              U.data_ptr(), U.stride(0), workspace.data_ptr(), workspace.numel(), payload.data_ptr(),
                              picks.data_ptr(), w_work.data_ptr(), None if flags is None else flags.data_ptr(),
                              _stream(stream)))
    return payload, picks, w_work


def iq_sqrt_diag(hess: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """sqrt of the diagonal of each [256, 256] block: fp32 [nblk * 256]."""
    lib = load_library()
    _need(hess, torch.float32, "hess")
    if not hess.is_contiguous() or hess.numel() % (256 * 256):
        raise IQError("hess must be contiguous [nblk, 256, 256]")
    nblk = hess.numel() // (256 * 256)
    if out is None:
        out = torch.empty(nblk * 256, dtype=torch.float32, device=hess.device)
    _check(lib.iq_sqrt_diag(hess.data_ptr(), nblk, out.data_ptr(), _stream(stream)))
    return out


PROBE_KINDS = {"ffma": 0, "ffma2": 1, "candidate_mix": 2, "candidate_mix_ffma2": 3}


def probe_fp32(kind: str, blocks: int, iters: int, out: torch.Tensor, stream=None) -> int:
    """Launch the FP32 issue-rate probe (include/iq_probe.h); returns the lane ops it performs."""
    lib = load_library()
    _need(out, torch.float32, "out")
    if out.numel() < blocks * 256:
        raise IQError("out must hold blocks * 256 floats")
    k = PROBE_KINDS[kind]
    if lib.iq_probe_fp32(k, blocks, iters, out.data_ptr(), _stream(stream)) != 0:
        raise IQError("iq_probe_fp32 failed")
    return blocks * 256 * iters * int(lib.iq_probe_fp32_ops_per_iter(k))


def probe_bulk_wait(src: torch.Tensor | None, arm: bool, limit_cycles: int, out: torch.Tensor, stream=None) -> None:
    """Launch the bulk-copy wait check (include/iq_probe.h): out[0] = 1 if the wait completed in
    time, out[1] = the weighted word sum of what was copied."""
    lib = load_library()
    _need(out, torch.int32, "out")
    nbytes = 0 if src is None else src.numel() * src.element_size()
    if lib.iq_probe_bulk_wait(None if src is None else src.data_ptr(), nbytes, int(arm), limit_cycles,
                              out.data_ptr(), _stream(stream)) != 0:
        raise IQError("iq_probe_bulk_wait failed")


def build_info() -> str:
    return load_library().iq_build_info().decode()
