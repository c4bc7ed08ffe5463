"""Shared helpers of the parity tests: run the oracle on the very inputs the
CUDA path gets, and compare.

Tolerance of the W4A16 linear layer (floating point): the reference Y_ref is
the oracle's fp64 product over the same dequantized weights, rounded once to
the output dtype (Y_ref_r).  The CUDA result Y must satisfy
    max |Y - Y_ref|              <= 1e-2 * max |Y_ref|
    sum |Y - Y_ref_r| / sum |Y_ref| <= 1e-3
Comparing with the rounded reference keeps the bound meaningful for bf16,
whose own output rounding alone is ~1.4e-3 relative on average.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MAX_REL = 1e-2
MEAN_REL = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a 16-bit float tensor (on the host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def odt(t: torch.Tensor) -> int:
    return oracle.F16 if t.dtype == torch.float16 else oracle.BF16


def oracle_quantize(W: torch.Tensor, group: int, sym: bool, col_scale=None):
    cs = None if col_scale is None else col_scale.detach().cpu().numpy().astype(np.float32)
    return oracle.quantize(bits(W), odt(W), group, sym, cs)


def round_to(y: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(y)).to(dtype).to(torch.float64).numpy()


def check_y(Y: torch.Tensor, Yref: np.ndarray, label: str = ""):
    """Assert the W4A16 tolerance; returns (max_rel, mean_rel) for reporting."""
    y = Y.detach().cpu().to(torch.float64).numpy()
    assert y.shape == Yref.shape, (y.shape, Yref.shape)
    assert np.isfinite(y).all(), f"{label}: non-finite output"
    yr = round_to(Yref, Y.dtype)
    amax = np.abs(Yref).max()
    max_err = np.abs(y - Yref).max()
    denom = np.abs(Yref).sum()
    mean_rel = np.abs(y - yr).sum() / denom if denom > 0 else np.abs(y - yr).sum()
    max_rel = max_err / amax if amax > 0 else max_err
    assert max_rel <= MAX_REL, f"{label}: max rel {max_rel:.3e}"
    assert mean_rel <= MEAN_REL, f"{label}: mean rel {mean_rel:.3e}"
    return max_rel, mean_rel


def oracle_linear(X: torch.Tensor, packed, scales, zeros, K: int, group: int = 128, rows=None):
    """fp64 Y_ref from the oracle for (optionally) a subset of weight rows n."""
    p = packed if isinstance(packed, np.ndarray) else packed.cpu().numpy()
    s = scales if isinstance(scales, np.ndarray) else scales.cpu().numpy()
    z = None if zeros is None else (zeros if isinstance(zeros, np.ndarray) else zeros.cpu().numpy())
    if rows is not None:
        p, s = p[rows], s[rows]
        z = None if z is None else z[rows]
    What = oracle.dequant(p, s, z, K, group)
    return oracle.linear(bits(X), odt(X), What)
