"""The FMA-pipe 2^x of csrc/ra_exp2.cuh, checked on the CPU: its constants
are what the committed Remez fit (csrc/fit_exp2_poly.py) produces, the
stated error bound holds for the cubic with float32 Horner evaluation, and a
float32 emulation of the whole exp2_poly2 algorithm (round-to-integer split,
cubic, exponent add) stays within that bound of 2^x over the range the
kernels feed it."""

from __future__ import annotations

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "ring_attention_ordered_b200", "csrc")


def _header_constants():
    text = open(os.path.join(CSRC, "ra_exp2.cuh")).read()
    vals = {int(m.group(1)): np.float32(float(m.group(2)))
            for m in re.finditer(r"EXP2_C(\d) = ([-+0-9.e]+)f;", text)}
    bound = float(re.search(r"max relative error ([0-9.e-]+)", text).group(1))
    return np.array([vals[i] for i in range(4)], dtype=np.float32), bound


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly",
                                                  os.path.join(CSRC, "fit_exp2_poly.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_constants_are_the_committed_fit():
    c_hdr, _ = _header_constants()
    fit = _fit_module()
    coef = fit.remez_relative(lambda t: np.exp2(t), -0.5, 0.5, 3).astype(np.float32)
    # the fit is deterministic; its float32 rounding is what the header holds
    # (printed with 10 significant digits, which round-trips float32)
    assert np.array_equal(coef, c_hdr), (coef, c_hdr)


def test_stated_bound_holds_for_float32_horner():
    c_hdr, bound = _header_constants()
    fit = _fit_module()
    f = np.linspace(-0.5, 0.5, 400001)
    rel = np.abs(fit.horner_f32(c_hdr, f).astype(np.float64) / np.exp2(f) - 1.0)
    assert rel.max() <= bound * 1.0001
    # and it is a minimax fit: the error reaches the bound, alternating
    assert rel.max() > 0.9 * bound


def _exp2_poly2_emulated(x, c):
    """float32 emulation of exp2_poly2 (separate multiply and add where the
    device fuses them: each step rounds at least as often as on the GPU)."""
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    j = (t - magic).astype(f32)
    f = (x - j).astype(f32)
    q = (c[3] * f + c[2]).astype(f32)
    q = (q * f + c[1]).astype(f32)
    q = (q * f + c[0]).astype(f32)
    bits = q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(f32)


def test_split_and_scale_reach_2_pow_x_within_the_bound():
    c_hdr, bound = _header_constants()
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-124.0, 8.5, 400000),
                        np.arange(-124, 9, dtype=np.float64) + 0.5,      # split ties
                        np.arange(-124, 9, dtype=np.float64)]).astype(np.float32)
    got = _exp2_poly2_emulated(x, c_hdr).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= bound * 1.05, rel.max()


def test_below_the_clamp_the_result_is_negligible():
    c_hdr, _ = _header_constants()
    got = _exp2_poly2_emulated(np.array([-200.0, -1e30, -126.0], dtype=np.float32), c_hdr)
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124)
