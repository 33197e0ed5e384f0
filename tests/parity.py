"""Comparison helpers shared by the GPU parity tests.

Tolerances (fp64 oracle vs the bf16-in / fp32-accumulate / bf16-out kernel):

* O: mean |err| <= 1e-3 over all compared elements, and per element
  |err| <= 1e-2, widened to one bf16 ulp of the oracle value where that ulp is
  larger (|O| >= 2): the output is stored in bf16, whose spacing there exceeds
  1e-2, so no bf16 value can be closer than half an ulp and fp32 accumulation
  error may round to the neighbouring value.
* LSE: max |err| <= 1e-3.
"""

from __future__ import annotations

import numpy as np
import torch

O_MAX = 1e-2
O_MEAN = 1e-3
LSE_MAX = 1e-3


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits)."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def o_bound(o_ref: np.ndarray) -> np.ndarray:
    return np.maximum(O_MAX, bf16_ulp(o_ref))


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what: str = ""):
    """Assert the tolerances above; return a dict of error statistics."""
    og, lg = to_np(o_gpu), to_np(lse_gpu)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse_ref = np.asarray(lse_ref, dtype=np.float64)
    assert og.shape == o_ref.shape, (og.shape, o_ref.shape)
    assert lg.shape == lse_ref.shape, (lg.shape, lse_ref.shape)
    assert np.all(np.isfinite(og)), f"{what}: non-finite O"
    assert np.all(np.isfinite(lg)), f"{what}: non-finite LSE"
    err = np.abs(og - o_ref)
    lerr = np.abs(lg - lse_ref)
    bound = o_bound(o_ref)
    stats = {
        "o_max": float(err.max()) if err.size else 0.0,
        "o_mean": float(err.mean()) if err.size else 0.0,
        "o_over_1e-2": int((err > O_MAX).sum()),
        "lse_max": float(lerr.max()) if lerr.size else 0.0,
        "n": int(err.size),
    }
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} O elements beyond bound; worst err {err[bad].max():.3e} "
        f"at ref {o_ref[bad][np.argmax(err[bad])]:.4f}; stats {stats}")
    assert stats["o_mean"] <= O_MEAN, f"{what}: mean |err| {stats['o_mean']:.3e}; {stats}"
    assert stats["lse_max"] <= LSE_MAX, f"{what}: LSE err {stats['lse_max']:.3e}; {stats}"
    return stats


# Gradients (fp64 oracle vs the backward kernels: bf16 inputs, P and dS
# rounded to bf16 before their products, fp32 accumulation, bf16 outputs).
# Each element carries the bf16 rounding of its own value (2^-9 relative) and
# of the terms it sums (P and dS, 2^-9 relative each, with partial
# cancellation in dK and dQ, whose terms sum to zero over keys); measured
# against the scale of the tensor:
#   max |err| <= GRAD_MAX * max |ref| + GRAD_ATOL
#   mean |err| <= GRAD_MEAN * mean |ref| + GRAD_ATOL
# GRAD_ATOL covers a gradient that is exactly zero by cancellation (one key
# per row: dS = P (dP - D) with dP and D the same dot product of O(1) unit
# normal terms, summed in a different order in fp32, ~1e-6 apart).
GRAD_MAX = 2.0 ** -6
GRAD_MEAN = 2.0 ** -8
GRAD_ATOL = 1e-5


def compare_grad(g_gpu, g_ref, what: str = ""):
    """Assert the gradient tolerances above; return error statistics."""
    g, r = to_np(g_gpu), np.asarray(g_ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite gradient"
    err = np.abs(g - r)
    scale_max = float(np.abs(r).max()) if r.size else 0.0
    scale_mean = float(np.abs(r).mean()) if r.size else 0.0
    stats = {
        "max_err": float(err.max()) if err.size else 0.0,
        "mean_err": float(err.mean()) if err.size else 0.0,
        "max_ref": scale_max,
        "mean_ref": scale_mean,
    }
    assert stats["max_err"] <= GRAD_MAX * scale_max + GRAD_ATOL, f"{what}: max {stats}"
    assert stats["mean_err"] <= GRAD_MEAN * scale_mean + GRAD_ATOL, f"{what}: mean {stats}"
    return stats
