"""FP8 (E4M3) block quantisation and the attention it stands for: a plain
CPU restatement (slow).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the CPU
baseline of the benchmark, never by the product path.

The FlashAttention article (developer.aliyun page, section 二,
"FlashAttention-3 改进") says the FP8 forward runs its GEMMs on FP8 tensor
cores and keeps the precision loss down with block quantisation and an
"incoherent processing" step.  Readings taken here (each the plainest one the
page supports; the page gives no formula):

* Format: E4M3 of the OCP 8-bit floating-point specification, the variant
  FP8 tensor cores take: a sign bit, 4 exponent bits with bias 7, 3 mantissa
  bits, subnormals at exponent field 0, largest finite value 448, no
  infinities, and S.1111.111 as NaN.
* Block: the 128-row tile of one (batch, head) -- the tile the attention
  kernels already work on.  scale = amax / 448 in float32, amax taken over
  the tile's rows and all d columns; an all-zero tile gets scale 1.  Each
  element x becomes e4m3(x / scale): the quotient is rounded to float32, then
  to E4M3 by round to nearest, ties to even, with magnitudes above 448
  saturated to 448.  When L is not a multiple of 128 the last block holds the
  remaining rows.
* The attention the FP8 path approximates is exact attention (``attn_fp64``)
  of the dequantised tensors code * scale.
* Incoherent processing is not restated: the page names it without defining
  it.
"""

from __future__ import annotations

import numpy as np

from .attn_fp64 import attention, attention_rows

E4M3_MAX = 448.0
E4M3_BIAS = 7
E4M3_MANT_BITS = 3
BLOCK = 128


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 code (uint8) as float64, from the bit fields:
    exponent field e, mantissa field m; e = 0 gives m * 2^-9 (subnormal),
    otherwise (1 + m/8) * 2^(e-7); e = 15 with m = 7 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> E4M3_MANT_BITS) & 0xF
    m = c & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e - E4M3_BIAS)
    sub = m * 2.0 ** (1 - E4M3_BIAS - E4M3_MANT_BITS)
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, val)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 code of each value: round to nearest, ties to even, magnitudes
    above 448 saturated to 448, NaN to the NaN code.

    For |x| in the binade [2^e, 2^(e+1)) (e >= -6) the representable values
    are 2^(e-3) apart; below 2^-6 (subnormals) they are 2^-9 apart.  |x| is
    divided by that spacing (exact: a power of two), rounded half to even
    (numpy's rint), and the result is written back into the bit fields."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, E4M3_MAX))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, 1 - E4M3_BIAS)                     # subnormals share 2^-6's spacing
    quantum = np.exp2(e - E4M3_MANT_BITS)
    v = np.rint(a / quantum) * quantum                   # rint: half to even
    v = np.minimum(v, E4M3_MAX)                          # 448 is finite; nothing rounds past it
    # bit fields of the rounded value
    with np.errstate(divide="ignore"):
        ev = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    is_sub = v < 2.0 ** (1 - E4M3_BIAS)
    exp_field = np.where(is_sub, 0, ev + E4M3_BIAS)
    mant = np.where(is_sub, v / 2.0 ** (1 - E4M3_BIAS - E4M3_MANT_BITS),
                    (v / np.exp2(ev) - 1.0) * 8.0)
    code = (exp_field.astype(np.int64) << E4M3_MANT_BITS) | np.rint(mant).astype(np.int64)
    code = np.where(nan, 0x7F, code) | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def _f32(x) -> np.ndarray:
    if hasattr(x, "detach") and hasattr(x, "float"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float32)


def quantize_blocks(x, block: int = BLOCK):
    """Block quantisation of x [B, L, H, d] (any real dtype whose values
    float32 holds exactly, such as bf16).

    Returns ``codes`` uint8 [B, L, H, d] and ``scales`` float32 [B, H, T],
    T = ceil(L / block): tile t of head h holds rows [t*block, (t+1)*block).
    """
    x32 = _f32(x)
    if x32.ndim != 4:
        raise ValueError("x must be [B, L, H, d]")
    B, L, H, d = x32.shape
    T = -(-L // block)
    codes = np.empty((B, L, H, d), dtype=np.uint8)
    scales = np.empty((B, H, T), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                tile = x32[b, t * block:(t + 1) * block, h, :]
                amax = np.float32(np.abs(tile).max()) if tile.size else np.float32(0)
                s = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))
                scales[b, h, t] = s
                codes[b, t * block:(t + 1) * block, h, :] = e4m3_encode(
                    (tile / s).astype(np.float32))
    return codes, scales


def dequantize_blocks(codes, scales, block: int = BLOCK) -> np.ndarray:
    """code * scale of the code's tile, as float64 [B, L, H, d] (exact)."""
    codes = np.asarray(codes)
    scales = np.asarray(scales, dtype=np.float64)
    B, L, H, d = codes.shape
    vals = e4m3_decode(codes)
    tile_of_row = np.arange(L) // block
    # scales [B, H, T] -> per row [B, L, H, 1]
    per_row = scales[:, :, tile_of_row].transpose(0, 2, 1)[..., None]
    return vals * per_row


class DequantView:
    """Read-only view of dequantised values indexed like the [B, L, H, d]
    tensor they stand for, decoding only the slice asked for (the large
    workloads do not fit in memory as float64)."""

    def __init__(self, codes, scales, block: int = BLOCK):
        self.codes = np.asarray(codes)
        self.scales = np.asarray(scales, dtype=np.float64)
        self.block = block
        self.shape = self.codes.shape
        self.ndim = 4

    def __getitem__(self, idx):
        b, rows, h, cols = idx
        c = self.codes[b, rows, h, cols]
        r = np.arange(self.shape[1])[rows]
        s = self.scales[b, h, r // self.block]
        return e4m3_decode(c) * np.asarray(s)[..., None]


def attention_fp8(q8, sq, k8, sk, v8, sv, causal: bool, scale: float):
    """Exact attention of the dequantised tensors: O [B, L, Hq, d] and
    lse [B, Hq, L] in float64 (the definition of ``attn_fp64.attention``)."""
    return attention(dequantize_blocks(q8, sq), dequantize_blocks(k8, sk),
                     dequantize_blocks(v8, sv), causal, scale)


def attention_fp8_rows(q8, sq, k8, sk, v8, sv, causal: bool, scale: float, bhr):
    """:func:`attention_fp8` for the listed (b, h, r) rows only."""
    return attention_rows(DequantView(q8, sq), DequantView(k8, sk), DequantView(v8, sv),
                          causal, scale, bhr)
