"""Seeded synthetic inputs for the IQ encoder path.

This module only draws random numbers: codebook grids, bf16 weights, per-column importance and
block Hessians. It holds none of the encoder's arithmetic, so both the CUDA path and the CPU oracle
take their inputs from here without sharing any of the method.

Recipes (all seeded, all reproducible):

* IQ1_S grid: 2048 distinct 8-vectors over {-1, 0, 1}, coordinates i.i.d. uniform, duplicates
  rejected in draw order. The real GGML tables are third-party data and are not used.
* IQ2_XS grid: 512 distinct 8-vectors over {1, 3, 5, 7}, drawn the same way.
* Weights: i.i.d. normal in fp32, rounded to bf16 (round to nearest even). Outlier columns are
  scaled by 8 after the rounding, which is exact in bf16. A stack of expert weights draws expert e
  from its own CPU generator (seed * 1024 + e), so any expert can be rebuilt on the host alone.
* Importance: per input column, log-normal(0, 1) in fp64, stored as fp32; the square-root
  variant is the square root of a log-normal Hessian diagonal.
* Block Hessian: H = U^-1 U^-T for an upper-triangular U with diagonal uniform in [0.5, 2] and
  off-diagonal N(0, 0.02^2), computed in fp64, symmetrised, stored as fp32.
"""

from __future__ import annotations

import numpy as np
import torch

GRID_SEED = 0x16C0DE
BLOCK = 256

IQ1S_GRID_ENTRIES = 2048
IQ2XS_GRID_ENTRIES = 512
IQ2S_GRID_ENTRIES = 1024


def _distinct_rows(values: np.ndarray, n: int, seed: int) -> np.ndarray:
    """Draw n distinct 8-vectors whose coordinates are uniform over `values`."""
    rng = np.random.Generator(np.random.PCG64(seed))
    seen: set[bytes] = set()
    rows: list[np.ndarray] = []
    while len(rows) < n:
        batch = values[rng.integers(0, len(values), size=(4 * n, 8))]
        for r in batch:
            key = r.tobytes()
            if key in seen:
                continue
            seen.add(key)
            rows.append(r)
            if len(rows) == n:
                break
    return np.ascontiguousarray(np.stack(rows).astype(np.int8))


def iq1s_grid(seed: int = GRID_SEED) -> np.ndarray:
    """[2048, 8] int8, entries in {-1, 0, 1}, all rows distinct."""
    return _distinct_rows(np.array([-1, 0, 1], dtype=np.int8), IQ1S_GRID_ENTRIES, seed)


def iq2xs_grid(seed: int = GRID_SEED + 1) -> np.ndarray:
    """[512, 8] int8, entries in {1, 3, 5, 7}, all rows distinct."""
    return _distinct_rows(np.array([1, 3, 5, 7], dtype=np.int8), IQ2XS_GRID_ENTRIES, seed)


def iq2s_grid(seed: int = GRID_SEED + 2) -> np.ndarray:
    """[1024, 8] int8, entries in {1, 3, 5, 7}, all rows distinct."""
    return _distinct_rows(np.array([1, 3, 5, 7], dtype=np.int8), IQ2S_GRID_ENTRIES, seed)


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """i.i.d. N(0, std^2) drawn in fp32 on `device`, rounded to bf16."""
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def normal_bf16_experts(experts: int, rows: int, cols: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """[experts, rows, cols] bf16: expert e is normal_bf16((rows, cols), std, seed * 1024 + e) drawn
    on the host, then moved to `device` one expert at a time."""
    out = torch.empty((experts, rows, cols), dtype=torch.bfloat16, device=device)
    for e in range(experts):
        out[e].copy_(expert_bf16(e, rows, cols, std, seed))
    return out


def expert_bf16(e: int, rows: int, cols: int, std: float, seed: int) -> torch.Tensor:
    """Expert e of normal_bf16_experts, on the host."""
    return normal_bf16((rows, cols), std, seed * 1024 + e)


def outlier_columns(cols: int, frac: float, seed: int) -> torch.Tensor:
    """A seeded choice of round(frac * cols) column indices."""
    g = torch.Generator().manual_seed(seed)
    n = int(round(frac * cols))
    return torch.randperm(cols, generator=g)[:n].sort().values


def with_outlier_columns(w: torch.Tensor, cols_idx: torch.Tensor, factor: float = 8.0) -> torch.Tensor:
    """Scale the chosen columns by a power of two (exact in bf16)."""
    w = w.clone()
    w[..., cols_idx.to(w.device)] *= factor
    return w


def lognormal(shape, seed: int, device="cpu") -> torch.Tensor:
    """log-normal(0, 1) values drawn in fp64, stored as fp32."""
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(shape, generator=g, dtype=torch.float64)
    return torch.exp(z).to(torch.float32).to(device)


def sqrt_lognormal(shape, seed: int, device="cpu") -> torch.Tensor:
    """Square root of a log-normal(0, 1) Hessian diagonal, fp64 then fp32."""
    g = torch.Generator().manual_seed(seed)
    z = torch.randn(shape, generator=g, dtype=torch.float64)
    return torch.sqrt(torch.exp(z)).to(torch.float32).to(device)


def block_factor(seed: int, n: int = BLOCK, offdiag_std: float = 0.02) -> torch.Tensor:
    """Upper-triangular U (fp64 [n, n]): diagonal uniform in [0.5, 2], above it N(0, std^2)."""
    g = torch.Generator().manual_seed(seed)
    diag = 0.5 + 1.5 * torch.rand(n, generator=g, dtype=torch.float64)
    off = offdiag_std * torch.randn((n, n), generator=g, dtype=torch.float64)
    return torch.triu(off, diagonal=1) + torch.diag(diag)


def block_hessian(seed: int, n: int = BLOCK, offdiag_std: float = 0.02) -> torch.Tensor:
    """H = U^-1 U^-T (fp64, symmetrised) as fp32 [n, n], U = block_factor(seed)."""
    u = block_factor(seed, n, offdiag_std)
    uinv = torch.linalg.solve_triangular(u, torch.eye(n, dtype=torch.float64), upper=True)
    h = uinv @ uinv.T
    h = 0.5 * (h + h.T)
    return h.to(torch.float32).contiguous()


# ---------------------------------------------------------------------------------------------
# The five workloads. Each returns a dict of host (or `device`) tensors; names say what they are.
# ---------------------------------------------------------------------------------------------

def workload_iq1s_64x256(device="cpu"):
    """IQ1_S, one 64x256 bf16 weight N(0, 0.02^2), uniform importance."""
    return {
        "fmt": "iq1_s",
        "w": normal_bf16((64, 256), 0.02, 1001, device),
        "importance": None,
    }


def workload_iq1s_4096x4096_weighted(device="cpu", rows=4096, cols=4096):
    """IQ1_S weighted: N(0, 0.02^2) with 1% of columns x8, importance = sqrt(log-normal)."""
    w = normal_bf16((rows, cols), 0.02, 1002, device)
    w = with_outlier_columns(w, outlier_columns(cols, 0.01, 2002))
    return {"fmt": "iq1_s", "w": w, "importance": sqrt_lognormal((cols,), 3002, device)}


def workload_iq2xs_8192x4096(device="cpu", rows=8192, cols=4096):
    """IQ2_XS: N(0, 0.015^2), per-column log-normal importance."""
    return {
        "fmt": "iq2_xs",
        "w": normal_bf16((rows, cols), 0.015, 1003, device),
        "importance": lognormal((cols,), 3003, device),
    }


def workload_iq1s_moe(device="cpu", experts=256, rows=1536, cols=4096):
    """MoE batch: `experts` weights of rows x cols, N(0, 0.02^2), each expert drawn on the host from
    its own seed (1004 * 1024 + e); per-expert log-normal importance."""
    return {
        "fmt": "iq1_s",
        "w": normal_bf16_experts(experts, rows, cols, 0.02, 1004, device),
        "importance": lognormal((experts, cols), 3004, device),
    }


def workload_choice_iq2xs(device="cpu", rows=4096, cols=4096):
    """Local-Hessian choice search: N(0, 0.02^2) weight, one H per 256-column block."""
    nblk = cols // BLOCK
    hess = torch.stack([block_hessian(5000 + b) for b in range(nblk)]).to(device)
    return {"fmt": "iq2_xs", "w": normal_bf16((rows, cols), 0.02, 1005, device), "hess": hess}


def inverse_hessian_factor(nblk: int, seed: int = 5000, offdiag_std: float = 0.02, cross_seed: int = 7000,
                           cross_std: float = 0.02) -> torch.Tensor:
    """The upper Cholesky factor U of a weight's inverse Hessian (H^-1 = U^T U), fp32 [256 nblk]^2:
    diagonal block b is block_factor(seed + b), so that block b's local Hessian U_bb^-1 U_bb^-T is
    block_hessian(seed + b); the blocks above the diagonal are N(0, cross_std^2) (seed cross_seed),
    the ones below it zero."""
    n = nblk * BLOCK
    u = torch.zeros((n, n), dtype=torch.float64)
    g = torch.Generator().manual_seed(cross_seed)
    for b in range(nblk):
        s = slice(b * BLOCK, (b + 1) * BLOCK)
        u[s, s] = block_factor(seed + b, offdiag_std=offdiag_std)
        if b + 1 < nblk:
            u[s, (b + 1) * BLOCK:] = cross_std * torch.randn((BLOCK, n - (b + 1) * BLOCK), generator=g,
                                                             dtype=torch.float64)
    return u.to(torch.float32).contiguous()


def workload_gptq_iq2xs(device="cpu", rows=4096, cols=4096):
    """The per-block calibration loop: the local-Hessian workload's weight and block Hessians,
    plus the full inverse-Hessian factor U whose diagonal blocks give those Hessians."""
    wl = workload_choice_iq2xs(device, rows, cols)
    wl["U"] = inverse_hessian_factor(cols // BLOCK).to(device)
    return wl


def workload_choice_moe(device="cpu", experts=16, rows=1536, cols=4096):
    """Local-Hessian choice search over a stack of expert weights [experts, rows, cols], N(0, 0.02^2),
    each expert with its own H per 256-column block ([experts, nblk, 256, 256])."""
    nblk = cols // BLOCK
    hess = torch.stack([torch.stack([block_hessian(6000 + nblk * e + b) for b in range(nblk)])
                        for e in range(experts)]).to(device)
    return {"fmt": "iq2_xs", "w": normal_bf16((experts, rows, cols), 0.02, 1006, device), "hess": hess}
