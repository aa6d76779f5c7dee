"""Helpers shared by the GPU parity tests: input casting, the tolerance of the GEMM
contract, and sample selection. Holds no GEMM arithmetic of its own."""
from __future__ import annotations

import numpy as np
import torch

import oracle

TORCH_TO_ORC = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float16: oracle.F16}


def to_dtype(x: np.ndarray, dt: torch.dtype) -> torch.Tensor:
    """float32 numpy -> CPU torch tensor of dtype dt (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(dt)


def orc_view(t: torch.Tensor):
    """(numpy array, oracle dtype code) viewing a CPU tensor's storage; keeps strides."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        a = t.view(torch.int16).numpy().view(np.uint16)
        return a, oracle.BF16
    return t.numpy(), TORCH_TO_ORC[t.dtype]


def ulp_of(x: np.ndarray, dt: torch.dtype) -> np.ndarray:
    """Spacing of the output type at |x| (subnormal spacing below the smallest normal)."""
    prec, emin = {torch.float32: (24, -126), torch.bfloat16: (8, -126), torch.float16: (11, -14)}[dt]
    a = np.abs(x)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** emin)))
    return 2.0 ** (e - (prec - 1))


def check_tolerance(got: np.ndarray, ref: np.ndarray, absacc: np.ndarray, out_dt: torch.dtype,
                    rel: float = 1e-3, diag: float = 1e-4, what: str = ""):
    """|C - C_ref| <= rel * sum_k |a||b| + ulp_out(C_ref), and the excess over one ulp is
    at most diag * sum_k |a||b| (a far tighter check that FP32 accumulation meets)."""
    got = got.astype(np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    u = ulp_of(ref, out_dt)
    bound = rel * absacc + u
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} outside the bound; first at {tuple(i)}: got "
                             f"{got[tuple(i)]}, ref {ref[tuple(i)]}, bound {bound[tuple(i)]}")
    excess = np.maximum(err - u, 0.0) / np.maximum(absacc, 1e-30)
    assert excess.max() <= diag, f"{what}: excess/sum|a||b| = {excess.max():.3g}"
    return float(excess.max())


def sample_indices(n: int, tile: int, per_tile: int, seed: int) -> np.ndarray:
    """Indices covering every tile of a dimension (first/last row of each tile, the
    ragged tail and random picks)."""
    rs = np.random.RandomState(seed)
    idx = set()
    for t0 in range(0, n, tile):
        t1 = min(n, t0 + tile)
        idx.update({t0, t1 - 1})
        idx.update(rs.randint(t0, t1, size=min(per_tile, t1 - t0)).tolist())
    return np.array(sorted(idx), dtype=np.int64)
