"""Tolerance of the FP8 forward, derived from its arithmetic.

The FP8 kernel computes exact products of E4M3 codes accumulated in fp32
(scores), multiplies by the per-tile scales, and keeps fp32 softmax
statistics.  The only coarse rounding is of the probabilities: before the
P V product each weight p' = 2^(x - m) * f is rounded to E4M3, where m is the
row's reference maximum (log2 units, at most the true maximum, lagging it by
at most 8) and f = sv_j / R folds tile j's V scale into P (R = the largest V
scale of the head).  The row sum uses the unrounded p.

E4M3 rounding of a value y errs by at most 2^-4 * y in the normal range
(y >= 2^-6) and by at most 2^-10 below it (subnormal spacing 2^-9).  Mapped
to the normalised weight w_c = exp(s_c - lse) of key c, the error of key c's
contribution is at most

    dw_c = 2^-4 * w_c + 2^-10 / (f_c * l_M),   l_M = sum_c exp(s_c - max_c s_c),

since the lagging reference only shrinks the absolute term (its rescale
factor is <= 1 and the kernel's row sum is >= l_M).  Hence per output
element

    |O_gpu - O| <= sum_c dw_c |v_c|  (+ bf16 storage: 2^-9 |O|)
                   (+ fp32 score/sum rounding: 1e-3 * sum_c w_c |v_c|),

and, for the mean over elements, the root-sum-square of the same terms
bounds the expected error of a sum of independent zero-mean roundings.

The bounds use R over every tile of the head, which is at least the R any
kernel schedule takes, so they hold for either choice.
"""

from __future__ import annotations

import numpy as np

from oracle.fp8_fp64 import BLOCK, DequantView

LSE_MAX = 1e-3
REL_NORMAL = 2.0 ** -4
ABS_SUBNORMAL = 2.0 ** -10
BF16_HALF_ULP = 2.0 ** -9
FP32_SLACK = 1e-3


def bounds_from_scores(s, vv, f, rel_normal: float = REL_NORMAL,
                       abs_subnormal: float = ABS_SUBNORMAL):
    """Exact O and lse of score rows ``s`` [n, keys] (natural log, -inf for
    masked keys) against dequantised values ``vv`` [keys, d], with the bounds
    of the module docstring; ``f`` [keys] is each key's V-scale fraction
    sv_j / R.  Returns (o, lse, bmax, brms, slack)."""
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    lm = e.sum(axis=1, keepdims=True)
    w = e / lm
    dw = rel_normal * w + np.where(np.isfinite(s), abs_subnormal / (f[None, :] * lm), 0.0)
    return (w @ vv, (mx + np.log(lm))[:, 0], dw @ np.abs(vv), np.sqrt((dw * dw) @ (vv * vv)),
            FP32_SLACK * (w @ np.abs(vv)))


def fp8_reference(q8, sq, k8, sk, v8, sv, causal: bool, scale: float, bhr=None,
                  rel_normal: float = REL_NORMAL, abs_subnormal: float = ABS_SUBNORMAL,
                  row_block: int = 256):
    """Oracle O and lse of the dequantised tensors for the rows ``bhr``
    ([n, 3] of (b, h, r); every row when None), with the per-element bounds
    ``bmax`` (worst case) and ``brms`` (root sum of squares).

    Returns a dict of arrays shaped [n, d] (O, bounds) and [n] (lse), in the
    order of ``bhr`` (for every row: b-major, then h, then r)."""
    q = DequantView(q8, sq)
    k = DequantView(k8, sk)
    v = DequantView(v8, sv)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    if bhr is None:
        bb, hh, rr = np.meshgrid(np.arange(B), np.arange(Hq), np.arange(L), indexing="ij")
        bhr = np.stack([bb.ravel(), hh.ravel(), rr.ravel()], axis=1)
    bhr = np.asarray(bhr, dtype=np.int64).reshape(-1, 3)
    n = bhr.shape[0]
    out = {key: np.empty((n, d)) for key in ("o", "bmax", "brms", "slack")}
    out["lse"] = np.empty(n)
    sv = np.asarray(sv, dtype=np.float64)
    keys = bhr[:, 0] * Hq + bhr[:, 1]
    for key in np.unique(keys):
        b, h = int(key // Hq), int(key % Hq)
        kh = h // g
        idx = np.nonzero(keys == key)[0]
        kk = k[b, :, kh, :]
        vv = v[b, :, kh, :]
        f = sv[b, kh, np.arange(L) // BLOCK] / sv[b, kh].max()
        for s0 in range(0, len(idx), row_block):
            sel = idx[s0:s0 + row_block]
            rs = bhr[sel, 2]
            s = scale * (q[b, rs, h, :] @ kk.T)
            if causal:
                s[np.arange(L)[None, :] > rs[:, None]] = -np.inf
            o, lse, bmax, brms, slack = bounds_from_scores(s, vv, f, rel_normal, abs_subnormal)
            out["o"][sel], out["lse"][sel] = o, lse
            out["bmax"][sel], out["brms"][sel], out["slack"][sel] = bmax, brms, slack
    return out


def compare_fp8(o_gpu, lse_gpu, ref, what: str = ""):
    """Assert the bounds above on O (per element and in the mean) and
    |lse error| <= 1e-3; return error statistics.  ``o_gpu`` [n, d] and
    ``lse_gpu`` [n] in the order of the reference rows."""
    og = np.asarray(o_gpu, dtype=np.float64)
    lg = np.asarray(lse_gpu, dtype=np.float64)
    assert og.shape == ref["o"].shape and lg.shape == ref["lse"].shape
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg)), f"{what}: non-finite output"
    err = np.abs(og - ref["o"])
    store = BF16_HALF_ULP * np.abs(ref["o"])
    bound = ref["bmax"] + ref["slack"] + store + 1e-6
    lerr = np.abs(lg - ref["lse"])
    stats = {
        "o_max": float(err.max()), "o_mean": float(err.mean()),
        "bound_min": float(bound.min()), "rms_mean": float(ref["brms"].mean()),
        "lse_max": float(lerr.max()), "n": int(err.size),
    }
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} elements over the FP8 bound; worst excess "
        f"{float((err - bound).max()):.3e}; {stats}")
    mean_bound = float((ref["brms"] + ref["slack"] + store).mean()) + 1e-6
    assert err.mean() <= mean_bound, f"{what}: mean error {err.mean():.3e} > {mean_bound:.3e}; {stats}"
    assert lerr.max() <= LSE_MAX, f"{what}: lse error {lerr.max():.3e}; {stats}"
    return stats
