"""GPU parity of the FP8 path (through the C ABI): the block quantiser
bit for bit against the oracle's, and the FP8 forward against exact attention
of the oracle-dequantised tensors within the tolerance derived in
tests/parity_fp8.py.  The oracle quantises the bf16 inputs itself; nothing it
uses comes from the GPU."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from oracle.fp8_fp64 import quantize_blocks
from parity_fp8 import compare_fp8, fp8_reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


def _bf16(shape, seed, mult=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * mult).to(torch.bfloat16)


# ------------------------------------------------------------------ quantiser
def _all_magnitudes_case():
    """Tiles that hold every finite bf16 magnitude up to a chosen maximum,
    with both signs, each tile also holding that maximum (so it sets every
    tile's scale), for maxima at the edges of the quantiser's division: a
    scale amax / 448 that is subnormal (IEEE division path), barely normal,
    one and near the largest bf16."""
    bits = np.arange(0x8000, dtype=np.uint32)
    mags = (bits << 16).view(np.float32)
    mags = mags[np.isfinite(mags)]
    per_tile = 128 * 128 - 1
    tiles = []
    for target in (1e-37, 2.4e-35, 1.0, 3.0e38):
        amax = np.float32(torch.tensor(target).to(torch.bfloat16).float().item())
        m = np.sort(mags[mags <= amax])
        vals = np.concatenate([m, -m])
        vals = np.concatenate([vals, np.zeros(-vals.size % per_tile, dtype=np.float32)])
        for chunk in vals.reshape(-1, per_tile):
            tiles.append(np.concatenate([np.float32([amax]), chunk]).reshape(128, 128))
    x = np.concatenate(tiles)[None, :, None, :]
    xt = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xt.float(), torch.from_numpy(x))      # exact bf16 values
    return xt


def _quant_case(name):
    if name == "ragged_d64":
        return _bf16((1, 300, 2, 64), 1)
    if name == "zero_and_large_tiles":
        x = _bf16((2, 512, 3, 128), 2)
        x[1, 128:256, 2, :] = 0
        x[0, 384:512, 1, :] *= 300.0
        x[0, 5, 0, 7] = 1e-30        # far below E4M3's range after scaling
        return x
    if name == "d256_two_tiles":
        return _bf16((1, 130, 1, 256), 3, mult=1e-3)
    if name == "d8":
        return _bf16((1, 129, 2, 8), 4, mult=50.0)
    if name == "one_row":
        return _bf16((1, 1, 1, 16), 5)
    if name == "all_magnitudes":
        return _all_magnitudes_case()
    raise KeyError(name)


@pytest.mark.parametrize("name", ["ragged_d64", "zero_and_large_tiles", "d256_two_tiles", "d8",
                                  "one_row", "all_magnitudes"])
def test_quantize_matches_oracle_bitwise(ra, name):
    x = _quant_case(name)
    codes, scales = ra.quantize_fp8(x.cuda())
    ra.check_status()
    c_ref, s_ref = quantize_blocks(x)
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    c = codes.cpu().numpy()
    assert np.array_equal(c, c_ref), f"{int((c != c_ref).sum())} codes differ"


# ------------------------------------------------------------------ forward
def _oracle_inputs(q, k, v):
    return (*quantize_blocks(q), *quantize_blocks(k), *quantize_blocks(v))


def _gpu_fp8(api, q, k, v, n_ring, causal, scale):
    q8, sq = api.quantize_fp8(q.cuda())
    k8, sk = api.quantize_fp8(k.cuda())
    v8, sv = api.quantize_fp8(v.cuda())
    out, lse = api.fwd_fp8(q8, sq, k8, sk, v8, sv, n_ring, causal, scale)
    api.check_status()
    return out, lse


# (B, Hq, Hkv, L, n_ring, causal), d = 128: several tiles, ring sizes 1..16,
# GQA groups 1..4 (odd group included), blocks of one to several tiles
SMALL = [
    (1, 1, 1, 128, 1, True),
    (1, 2, 2, 512, 4, True),
    (1, 2, 2, 512, 4, False),
    (1, 8, 2, 1024, 2, True),
    (1, 3, 1, 512, 1, True),
    (2, 4, 4, 768, 3, False),
    (1, 6, 2, 256, 1, False),
    (1, 2, 2, 2048, 16, True),
    (3, 2, 2, 384, 3, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,L,n_ring,causal", SMALL)
def test_fwd_fp8_small_shapes(ra, B, Hq, Hkv, L, n_ring, causal):
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, L, 128, seed=7000 + B * 100 + L + n_ring)
    scale = 1.0 / math.sqrt(128)
    out, lse = _gpu_fp8(ra, q, k, v, n_ring, causal, scale)
    ref = fp8_reference(*_oracle_inputs(q, k, v), causal, scale)
    # reference rows are ordered b, h, r
    o_g = out.float().cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, 128)
    l_g = lse.cpu().numpy().reshape(-1)
    compare_fp8(o_g, l_g, ref, f"fp8 {B},{Hq},{Hkv},{L},{n_ring},{causal}")


def _head_subset(w):
    """Query heads whose rows are checked at full size, and their K/V heads:
    the first and the last K/V group, so GQA grouping is kept."""
    g = w.Hq // w.Hkv
    kvh = sorted({0, w.Hkv - 1})
    qh = [kh * g + i for kh in kvh for i in range(g)]
    return qh, kvh


@pytest.mark.parametrize("name,n_sample", [
    ("l8k_h8_causal", 2048),
    ("l32k_gqa4_causal", 1024),
    ("l128k_h32_causal", 512),
])
def test_fwd_fp8_workload_sampled_rows(ra, name, n_sample):
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    q8, sq = ra.quantize_fp8(qd)
    k8, sk = ra.quantize_fp8(kd)
    v8, sv = ra.quantize_fp8(vd)
    del qd, kd, vd
    out, lse = ra.fwd_fp8(q8, sq, k8, sk, v8, sv, w.n_ring, w.causal, w.scale)
    ra.check_status()

    # the oracle quantises the checked heads itself (scales are per head, so
    # a head subset quantises exactly as the whole tensor does)
    qh, kvh = _head_subset(w)
    q_s, k_s, v_s = q[:, :, qh].contiguous(), k[:, :, kvh].contiguous(), v[:, :, kvh].contiguous()
    o_in = _oracle_inputs(q_s, k_s, v_s)
    # the GPU's codes for those heads are the oracle's, bit for bit
    assert np.array_equal(k8[:, :, kvh].cpu().numpy(), o_in[2])
    assert np.array_equal(sv[:, kvh].cpu().numpy(), o_in[5])
    rng = np.random.default_rng(w.seed)
    n = min(n_sample, w.B * len(qh) * w.L)
    flat = rng.choice(w.B * len(qh) * w.L, size=n, replace=False)
    bhr = np.stack([flat // (len(qh) * w.L), (flat // w.L) % len(qh), flat % w.L], axis=1)
    blk = w.L // w.n_ring
    edges = np.array([[0, 0, 0], [0, 0, blk - 1], [0, 0, blk], [0, len(qh) - 1, w.L - 1]])
    bhr = np.concatenate([bhr, edges]).astype(np.int64)
    ref = fp8_reference(*o_in, w.causal, w.scale, bhr)
    hq = torch.tensor(qh)[torch.from_numpy(bhr[:, 1])].cuda()
    b = torch.from_numpy(bhr[:, 0]).cuda()
    r = torch.from_numpy(bhr[:, 2]).cuda()
    stats = compare_fp8(out[b, r, hq, :].float().cpu().numpy(), lse[b, hq, r].cpu().numpy(), ref,
                        name)
    # what FP8 costs against the exact bf16-input attention (reported, and
    # bounded loosely: a few percent of |v| at most)
    bhr_full = np.stack([bhr[:, 0], np.array(qh)[bhr[:, 1]], bhr[:, 2]], axis=1)
    o_true, _ = oracle.attention_rows(q, k, v, w.causal, w.scale, bhr_full)
    dev = np.abs(out[b, r, hq, :].float().cpu().numpy() - o_true)
    print(name, stats, "vs bf16-input attention: max", dev.max(), "mean", dev.mean())
    assert dev.mean() < 3e-2


def test_fwd_fp8_sink_workload_sampled_rows(ra):
    """The 1M-token GQA workload whose first four keys carry +3 (attention
    sinks: rows dominated by a few keys, where the E4M3 rounding of a large
    weight matters most), 128 rows drawn per head plus sink-dominated early
    rows and ring-block edges, against exact attention of the dequantised
    inputs.  The oracle quantises K and V whole and Q only in the 128-row
    tiles that hold checked rows (a tile's codes depend on that tile alone);
    the GPU's codes of those tiles must equal the oracle's bit for bit."""
    from oracle.fp8_fp64 import BLOCK
    from ring_attention_ordered_b200.inputs import WORKLOADS, sample_rows_per_head, workload_inputs
    w = WORKLOADS["l1m_gqa4_sink_causal"]
    q, k, v = workload_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    q8, sq = ra.quantize_fp8(qd)
    k8, sk = ra.quantize_fp8(kd)
    v8, sv = ra.quantize_fp8(vd)
    del qd, kd, vd
    out, lse = ra.fwd_fp8(q8, sq, k8, sk, v8, sv, w.n_ring, w.causal, w.scale)
    ra.check_status()
    blk = w.L // w.n_ring
    extra = np.array([[0, h, r] for h in (0, w.Hq - 1)
                      for r in (0, 3, 4, 5, 17, 127, 128, 1000, blk - 1, blk, w.L - 1)])
    bhr = np.concatenate([sample_rows_per_head(w, 128), extra]).astype(np.int64)
    k8o, sko = quantize_blocks(k)
    v8o, svo = quantize_blocks(v)
    assert np.array_equal(k8.cpu().numpy(), k8o) and np.array_equal(sk.cpu().numpy(), sko)
    assert np.array_equal(v8.cpu().numpy(), v8o) and np.array_equal(sv.cpu().numpy(), svo)
    q8o = np.zeros(tuple(q.shape), dtype=np.uint8)
    sqo = np.ones(tuple(sq.shape), dtype=np.float32)
    for b, h, t in sorted({(int(b), int(h), int(r) // BLOCK) for b, h, r in bhr}):
        c, sc = quantize_blocks(q[b:b + 1, t * BLOCK:(t + 1) * BLOCK, h:h + 1])
        q8o[b, t * BLOCK:(t + 1) * BLOCK, h] = c[0, :, 0]
        sqo[b, h, t] = sc[0, 0, 0]
    for b, h, t in sorted({(int(b), int(h), int(r) // BLOCK) for b, h, r in bhr}):
        assert np.array_equal(q8[b, t * BLOCK:(t + 1) * BLOCK, h].cpu().numpy(),
                              q8o[b, t * BLOCK:(t + 1) * BLOCK, h])
        assert float(sq[b, h, t]) == float(sqo[b, h, t])
    ref = fp8_reference(q8o, sqo, k8o, sko, v8o, svo, w.causal, w.scale, bhr, row_block=32)
    b, h, r = (torch.from_numpy(bhr[:, i]).cuda() for i in range(3))
    stats = compare_fp8(out[b, r, h, :].float().cpu().numpy(), lse[b, h, r].cpu().numpy(), ref,
                        w.name)
    o_true, _ = oracle.attention_rows(q, k, v, w.causal, w.scale, bhr, row_block=16)
    dev = np.abs(out[b, r, h, :].float().cpu().numpy() - o_true)
    print(w.name, stats, "vs bf16-input attention: max", dev.max(), "mean", dev.mean())
    assert dev.mean() < 3e-2


def test_fp8_bounded_wait_reports_timeout_and_recovers(ra):
    from ring_attention_ordered_b200 import _lib
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(1, 2, 2, 512, 128, seed=15)
    q8, sq = ra.quantize_fp8(q.cuda())
    k8, sk = ra.quantize_fp8(k.cuda())
    v8, sv = ra.quantize_fp8(v.cuda())
    ra.check_status()
    _lib.ring_attn_set_wait_limit_ns(50_000_000)
    _lib.ring_attn_debug_inject(1)
    try:
        ra.fwd_fp8(q8, sq, k8, sk, v8, sv, 4, True)
        with pytest.raises(_lib.RingAttnError) as e:
            ra.check_status()
        assert e.value.status == _lib.RA_ERR_TIMEOUT
    finally:
        _lib.ring_attn_debug_inject(0)
        _lib.ring_attn_set_wait_limit_ns(0)
    out, lse = ra.fwd_fp8(q8, sq, k8, sk, v8, sv, 4, True)
    ra.check_status()
    ref = fp8_reference(*_oracle_inputs(q, k, v), True, 1 / math.sqrt(128))
    compare_fp8(out.float().cpu().numpy().transpose(0, 2, 1, 3).reshape(-1, 128),
                lse.cpu().numpy().reshape(-1), ref, "after timeout")
