"""Pins of the FP8 oracle (oracle/fp8_fp64.py) against things other than
itself: the E4M3 bit-field definition, torch's float8_e4m3fn conversion (a
library routine), tie and saturation cases worked by hand, brute force on
tiny tiles, and a lossless case that reduces FP8 attention to the fp64
attention oracle.  Planted mistakes (mutants of the oracle) must fail."""

import math

import numpy as np
import pytest
import torch

from oracle import attention
from oracle.fp8_fp64 import (
    E4M3_MAX,
    DequantView,
    attention_fp8,
    attention_fp8_rows,
    dequantize_blocks,
    e4m3_decode,
    e4m3_encode,
    quantize_blocks,
)

ALL = np.arange(256, dtype=np.uint8)


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def _torch_encode(x32):
    return torch.from_numpy(np.asarray(x32, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


# ------------------------------------------------------------------ format
def test_decode_matches_torch_for_every_code():
    d = e4m3_decode(ALL)
    t = _torch_decode(ALL).astype(np.float64)
    assert np.array_equal(np.isnan(d), np.isnan(t))
    assert np.array_equal(d[~np.isnan(d)], t[~np.isnan(t)])
    # exactly two NaN codes (S.1111.111), no infinities
    assert sorted(ALL[np.isnan(d)].tolist()) == [0x7F, 0xFF]
    assert not np.isinf(d).any()


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x39, 1.125), (0x3F, 1.875), (0x40, 2.0), (0x7E, 448.0),
    (0xB8, -1.0), (0xFE, -448.0),
])
def test_decode_bit_fields(code, value):
    assert e4m3_decode(np.array([code], np.uint8))[0] == value


def test_encode_round_trips_every_finite_code():
    d = e4m3_decode(ALL)
    fin = ~np.isnan(d)
    assert np.array_equal(e4m3_encode(d[fin]), ALL[fin])


@pytest.mark.parametrize("x,code", [
    (1.0625, 0x38),            # tie between 1 (mantissa 000) and 1.125: even -> 1
    (1.1875, 0x3A),            # tie between 1.125 (001) and 1.25 (010): even -> 1.25
    (1.0625 + 1e-9, 0x39),     # just above the tie
    (2.0 ** -10, 0x00),        # tie between 0 and the smallest subnormal: 0
    (3 * 2.0 ** -10, 0x02),    # tie between 2^-9 (001) and 2^-8 (010): 2^-8
    (1.9375, 0x40),            # rounds up into the next binade
    (2.0 ** -6 - 2.0 ** -11, 0x08),  # rounds up out of the subnormals
    (448.0, 0x7E), (460.0, 0x7E), (480.0, 0x7E), (1e30, 0x7E),  # saturation
    (-1e30, 0xFE), (-0.0, 0x80),
])
def test_encode_ties_and_saturation(x, code):
    assert int(e4m3_encode(np.array([x]))[0]) == code


def test_encode_nan():
    c = int(e4m3_encode(np.array([np.nan]))[0])
    assert c & 0x7F == 0x7F


def test_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(300000) * np.exp2(rng.uniform(-14, 9, 300000))).astype(np.float32)
    x = x[np.abs(x) <= E4M3_MAX]
    assert np.array_equal(e4m3_encode(x.astype(np.float64)), _torch_encode(x))


def test_encode_error_within_half_spacing():
    rng = np.random.default_rng(1)
    x = rng.uniform(-448, 448, 100000)
    err = np.abs(e4m3_decode(e4m3_encode(x)) - x)
    a = np.abs(x)
    normal = a >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * a[normal])
    assert np.all(err[~normal] <= 2.0 ** -10)


def test_encode_mutant_truncation_fails():
    # a planted mistake: truncating instead of rounding to nearest
    def trunc(x):
        x = np.asarray(x, np.float64)
        e = np.maximum(np.floor(np.log2(np.maximum(np.abs(x), 1e-300))), -6)
        q = np.exp2(e - 3)
        return e4m3_encode(np.sign(x) * np.floor(np.abs(x) / q) * q)
    rng = np.random.default_rng(2)
    x = rng.uniform(-4, 4, 1000).astype(np.float32)
    assert not np.array_equal(trunc(x.astype(np.float64)), _torch_encode(x))


# ------------------------------------------------------------------ blocks
def _bf16(shape, seed, mult=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * mult).to(torch.bfloat16)


def test_quantize_brute_force_tiny():
    x = _bf16((1, 5, 2, 3), 3, mult=7.0)
    codes, scales = quantize_blocks(x, block=2)
    xf = x.float().numpy()
    assert scales.shape == (1, 2, 3)
    for h in range(2):
        for t in range(3):
            rows = range(2 * t, min(5, 2 * t + 2))
            amax = max(abs(float(xf[0, r, h, j])) for r in rows for j in range(3))
            s = np.float32(np.float32(amax) / np.float32(448.0))
            assert scales[0, h, t] == s
            for r in rows:
                for j in range(3):
                    q = float(np.float32(np.float32(xf[0, r, h, j]) / s))
                    # nearest E4M3 value by exhaustive search, ties to the even code
                    vals = e4m3_decode(ALL)
                    fin = ~np.isnan(vals)
                    dist = np.abs(vals[fin] - q)
                    best = ALL[fin][dist == dist.min()]
                    best = [c for c in best if (c & 1) == 0] or list(best)
                    if len(best) > 1:   # +0 and -0
                        best = [c for c in best if (c & 0x80) == (0x80 if q < 0 else 0)] or best
                    assert codes[0, r, h, j] == best[0], (r, h, j, q)


def test_quantize_amax_maps_to_448():
    x = _bf16((2, 256, 3, 64), 4, mult=3.0)
    codes, scales = quantize_blocks(x)
    vals = e4m3_decode(codes)
    for t in range(2):
        tile = np.abs(vals[:, t * 128:(t + 1) * 128])
        assert np.all(tile.max(axis=(1, 3)) == 448.0)


def test_quantize_error_bound_and_zero_tile():
    x = _bf16((1, 384, 2, 128), 5)
    x[:, 128:256, 1, :] = 0
    codes, scales = quantize_blocks(x)
    assert scales[0, 1, 1] == 1.0 and not codes[0, 128:256, 1, :].any()
    xd = dequantize_blocks(codes, scales)
    xf = x.double().numpy()
    s_row = scales[0][:, np.arange(384) // 128].T[None, :, :, None].astype(np.float64)
    err = np.abs(xd - xf)
    normal = np.abs(xf) >= 2.0 ** -6 * s_row
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(xf[normal]) * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * np.broadcast_to(s_row, err.shape)[~normal] * (1 + 1e-6))


def test_quantize_ragged_tail_and_tile_independence():
    x = _bf16((1, 300, 2, 64), 6)
    codes, scales = quantize_blocks(x)
    assert codes.shape == (1, 300, 2, 64) and scales.shape == (1, 2, 3)
    y = x.clone()
    y[:, 280, 0, 5] = 100.0      # only tile 2 of head 0 changes
    codes2, scales2 = quantize_blocks(y)
    assert np.array_equal(scales2[0, 0, :2], scales[0, 0, :2])
    assert np.array_equal(scales2[0, 1], scales[0, 1])
    assert scales2[0, 0, 2] == np.float32(np.float32(100.0) / np.float32(448.0))
    assert np.array_equal(codes2[:, :256], codes[:, :256])
    assert np.array_equal(codes2[:, 256:, 1], codes[:, 256:, 1])


def test_quantize_mutant_per_head_scale_fails():
    # a planted mistake: one scale per head over the whole sequence
    x = _bf16((1, 256, 1, 64), 7)
    x[:, :128] *= 8
    codes, scales = quantize_blocks(x)
    assert scales[0, 0, 0] > 4 * scales[0, 0, 1]
    whole = np.float32(np.abs(x.float().numpy()).max() / np.float32(448))
    assert scales[0, 0, 1] != whole


# ------------------------------------------------------------------ attention
def _grid_tensor(shape, seed, exp_shift):
    """Values on the E4M3 grid times 2^exp_shift, with one element of +-448
    per 128-row tile, so block quantisation is lossless."""
    rng = np.random.default_rng(seed)
    fin = ALL[(~np.isnan(e4m3_decode(ALL))) & (np.abs(e4m3_decode(ALL)) <= 64)]
    v = e4m3_decode(rng.choice(fin, size=shape))
    B, L, H, d = shape
    for t in range(0, L, 128):
        v[:, t, :, 0] = 448.0
    return torch.from_numpy(v * 2.0 ** exp_shift).to(torch.bfloat16)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_fp8_lossless_case_equals_fp64_attention(causal):
    q = _grid_tensor((1, 256, 4, 32), 8, -9)
    k = _grid_tensor((1, 256, 2, 32), 9, -8)
    v = _grid_tensor((1, 256, 2, 32), 10, -7)
    q8, sq = quantize_blocks(q)
    k8, sk = quantize_blocks(k)
    v8, sv = quantize_blocks(v)
    assert np.array_equal(dequantize_blocks(q8, sq), q.double().numpy())
    o8, l8 = attention_fp8(q8, sq, k8, sk, v8, sv, causal, 0.3)
    o, l_ = attention(q, k, v, causal, 0.3)
    assert np.max(np.abs(o8 - o)) < 1e-12 and np.max(np.abs(l8 - l_)) < 1e-12


def test_attention_fp8_mutant_missing_v_scale_fails():
    q = _grid_tensor((1, 128, 1, 16), 11, -9)
    k = _grid_tensor((1, 128, 1, 16), 12, -9)
    v = _grid_tensor((1, 128, 1, 16), 13, -7)
    q8, sq = quantize_blocks(q)
    k8, sk = quantize_blocks(k)
    v8, sv = quantize_blocks(v)
    o, _ = attention(q, k, v, False, 0.25)
    o_bad, _ = attention(dequantize_blocks(q8, sq), dequantize_blocks(k8, sk),
                         e4m3_decode(v8), False, 0.25)
    assert np.max(np.abs(o_bad - o)) > 1.0


def test_rows_and_view_agree_with_full():
    q = _bf16((2, 256, 4, 32), 14)
    k = _bf16((2, 256, 2, 32), 15)
    v = _bf16((2, 256, 2, 32), 16)
    q8, sq = quantize_blocks(q)
    k8, sk = quantize_blocks(k)
    v8, sv = quantize_blocks(v)
    view = DequantView(k8, sk)
    assert np.array_equal(view[1, :, 1, :], dequantize_blocks(k8, sk)[1, :, 1, :])
    o, l_ = attention_fp8(q8, sq, k8, sk, v8, sv, True, 1 / math.sqrt(32))
    bhr = np.array([[0, 0, 0], [1, 3, 255], [0, 2, 128], [1, 1, 7]])
    orow, lrow = attention_fp8_rows(q8, sq, k8, sk, v8, sv, True, 1 / math.sqrt(32), bhr)
    for i, (b, h, r) in enumerate(bhr):
        assert np.max(np.abs(orow[i] - o[b, r, h])) < 1e-12
        assert abs(lrow[i] - l_[b, h, r]) < 1e-12
