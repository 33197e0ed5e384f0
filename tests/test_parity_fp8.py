"""The FP8 tolerance (tests/parity_fp8.py) checked against an fp64 emulation
of the arithmetic it bounds: lazy reference maximum (moved only when a tile's
maximum exceeds it by more than 8 in log2 units), probabilities scaled by the
tile's V-scale fraction and rounded to E4M3 by the oracle's encoder, fp32-free
accumulation, and one division by the unrounded row sum at the end.  The
bound must hold on random, peaked, late-maximum and small-V-scale rows, and
weaker bounds (planted mistakes) must fail on some of them."""

import numpy as np
import pytest

from oracle.fp8_fp64 import e4m3_decode, e4m3_encode
from parity_fp8 import BF16_HALF_ULP, bounds_from_scores

TILE = 128


def _round_e4m3(y):
    return e4m3_decode(e4m3_encode(y))


def emulate_row(s, vcodes, sv_tile, order):
    """Rounded-P attention of one score row s [keys] (natural log, -inf for
    masked keys) against V codes [keys, d] whose tile j has scale sv_tile[j],
    visiting tiles in ``order``."""
    x = s / np.log(2.0)
    R = sv_tile.max()
    m, l_ = -np.inf, 0.0
    acc = np.zeros(vcodes.shape[1])
    for j in order:
        cols = np.arange(j * TILE, (j + 1) * TILE)
        xt = x[cols]
        mt = xt.max()
        if mt > m + 8:
            alpha = 0.0 if m == -np.inf else 2.0 ** (m - mt)
            acc *= alpha
            l_ *= alpha
            m = mt
        p = np.where(np.isfinite(xt), 2.0 ** (xt - m), 0.0)
        f = sv_tile[j] / R
        acc += _round_e4m3(p * f) @ vcodes[cols]
        l_ += p.sum()
    return acc * R / l_


def _case(kind, seed, n_tiles=8, d=16):
    rng = np.random.default_rng(seed)
    keys = n_tiles * TILE
    fin = np.arange(256, dtype=np.uint8)
    fin = fin[~np.isnan(e4m3_decode(fin))]
    vcodes = e4m3_decode(rng.choice(fin, size=(keys, d)))
    sv_tile = rng.uniform(0.5, 1.5, n_tiles) / 448.0
    s = rng.standard_normal(keys)
    order = list(range(n_tiles))
    if kind == "peaked":
        s[rng.choice(keys, 3, replace=False)] += 9.0
    elif kind == "late_max":
        # the maximum grows by less than 8 (log2) from tile to tile, so the
        # reference lags and scaled probabilities reach up to 2^8 f
        s = s * 0.3 + np.repeat(np.arange(n_tiles) * 4.0, TILE)
    elif kind == "small_v_scale":
        sv_tile[::2] *= 1e-3
    elif kind == "masked":
        s[keys // 2 + 7:] = -np.inf
    elif kind == "reverse":
        order = order[::-1]
    return s, vcodes, sv_tile, order


KINDS = ["random", "peaked", "late_max", "small_v_scale", "masked", "reverse"]


def _errors_and_bounds(kind, seed, **kw):
    s, vcodes, sv_tile, order = _case(kind, seed)
    vv = vcodes * np.repeat(sv_tile, TILE)[:, None]
    f = np.repeat(sv_tile / sv_tile.max(), TILE)
    o, lse, bmax, brms, slack = bounds_from_scores(s[None, :], vv, f, **kw)
    oe = emulate_row(s, vcodes, sv_tile, order)
    return np.abs(oe - o[0]), bmax[0], brms[0], slack[0], np.abs(o[0])


@pytest.mark.parametrize("kind", KINDS)
def test_bound_holds_on_emulated_rounding(kind):
    for seed in range(6):
        err, bmax, brms, slack, _ = _errors_and_bounds(kind, seed)
        assert np.all(err <= bmax + 1e-12), (kind, seed, float((err - bmax).max()))


def test_mean_error_within_rms_bound():
    errs, rms = [], []
    for kind in KINDS:
        for seed in range(6):
            err, bmax, brms, slack, _ = _errors_and_bounds(kind, seed)
            errs.append(err)
            rms.append(brms)
    assert np.mean(np.concatenate(errs)) <= np.mean(np.concatenate(rms))


def test_bound_is_not_vacuous():
    # the observed error reaches a fair share of the worst-case bound somewhere
    worst = 0.0
    for kind in KINDS:
        for seed in range(6):
            err, bmax, _, _, _ = _errors_and_bounds(kind, seed)
            worst = max(worst, float((err / bmax).max()))
    assert worst > 0.05


def test_weaker_bounds_fail():
    # planted mistakes in the tolerance: half the relative term, or no
    # subnormal term; each must be violated by some emulated row
    def violated(**kw):
        for kind in KINDS:
            for seed in range(6):
                err, bmax, _, _, _ = _errors_and_bounds(kind, seed, **kw)
                if np.any(err > bmax + 1e-12):
                    return True
        return False
    assert violated(abs_subnormal=0.0)
    # two keys, the second just under a rounding tie one binade up: its
    # rounding error is close to 2^-4 of its weight
    s = np.full(2 * TILE, -np.inf)
    s[0] = 0.0
    s[TILE] = np.log(1.0625 - 1e-4)
    vcodes = np.zeros((2 * TILE, 1))
    vcodes[TILE] = 1.0
    sv_tile = np.array([1.0, 1.0])
    oe = emulate_row(s, vcodes, sv_tile, [0, 1])
    vv = vcodes.copy()
    f = np.ones(2 * TILE)
    o, _, bmax_half, _, _ = bounds_from_scores(s[None, :], vv, f, rel_normal=2.0 ** -5,
                                               abs_subnormal=0.0)
    _, _, bmax_full, _, _ = bounds_from_scores(s[None, :], vv, f)
    err = abs(oe[0] - o[0, 0])
    assert err > bmax_half[0, 0]
    assert err <= bmax_full[0, 0]


def test_storage_term_is_half_a_bf16_ulp():
    assert BF16_HALF_ULP == 2.0 ** -9
