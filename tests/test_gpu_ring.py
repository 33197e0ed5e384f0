"""GPU parity of the per-visit entry point (ring_attn_fwd_visit, through the C
ABI) and of the ring's visit chain on one device, against the fp64 oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from parity import compare, to_np

pytestmark = pytest.mark.gpu

KIND = {0: "full", 1: "masked", 2: "strict"}


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


def visit(api, q, k, v, mask, fold=False, o_acc=None, lse_acc=None, with_out=True, scale=None):
    B, l, Hq, d = q.shape
    if o_acc is None:
        o_acc = torch.full((B, l, Hq, d), float("nan"), dtype=torch.float32, device="cuda")
        lse_acc = torch.full((B, Hq, l), float("nan"), dtype=torch.float32, device="cuda")
    out = torch.empty((B, l, Hq, d), dtype=torch.bfloat16, device="cuda") if with_out else None
    api.fwd_visit(q, k, v, o_acc, lse_acc, mask, fold, scale, out)
    api.check_status()
    return o_acc, lse_acc, out


def compare_partial(o, lse, o_ref, l_ref, what):
    """Parity of a partial result: rows the mask leaves empty must be exactly
    o = 0, lse = -inf; the others within the usual tolerances."""
    o, lse = to_np(o), to_np(lse)
    empty = np.isneginf(l_ref)                       # [B, Hq, l]
    assert np.array_equal(np.isneginf(lse), empty), what
    e = empty.transpose(0, 2, 1)                     # [B, l, Hq]
    assert np.all(o[e] == 0.0), what
    if (~empty).any():
        compare(o[~e], lse[~empty], o_ref[~e], l_ref[~empty], what)


# (B, Hq, Hkv, l, d): several tiles, a ragged tail, GQA, a one-row block
VISIT_SHAPES = [
    (1, 2, 2, 256, 128),
    (2, 4, 2, 200, 64),
    (1, 4, 1, 384, 128),
    (1, 3, 3, 130, 128),
    (1, 2, 1, 1, 128),
]


@pytest.mark.parametrize("mask", [0, 1, 2])
@pytest.mark.parametrize("B,Hq,Hkv,l,d", VISIT_SHAPES)
def test_visit_matches_oracle(ra, B, Hq, Hkv, l, d, mask):
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, l, d, seed=100 + l + d + mask)
    o_acc, lse_acc, out = visit(ra, q.cuda(), k.cuda(), v.cuda(), mask)
    o_ref, l_ref = oracle.block_attention(q, k, v, 1.0 / d ** 0.5, KIND[mask])
    compare_partial(o_acc, lse_acc, o_ref, l_ref, f"visit {(B, Hq, Hkv, l, d, mask)}")
    # out is the bf16 rounding of the accumulator, element for element
    assert torch.equal(out, o_acc.to(torch.bfloat16))


@pytest.mark.parametrize("mask_a,mask_b", [(1, 0), (0, 0), (1, 2), (2, 1)])
def test_fold_is_bitwise_the_merge_kernel(ra, mask_a, mask_b):
    """A folding visit gives bitwise what a fresh visit plus ring_attn_merge
    give, including the empty rows of a strict visit."""
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k1, v1 = (t.cuda() for t in make_inputs(2, 4, 2, 320, 128, seed=31))
    _, k2, v2 = (t.cuda() for t in make_inputs(2, 4, 2, 320, 128, seed=32))
    o_a, l_a, _ = visit(ra, q, k1, v1, mask_a)
    o_keep, l_keep = o_a.clone(), l_a.clone()
    o_f, l_f, out_f = visit(ra, q, k2, v2, mask_b, fold=True, o_acc=o_a, lse_acc=l_a)
    o_b, l_b, _ = visit(ra, q, k2, v2, mask_b)
    rows = 2 * 320 * 4
    # merge works on [rows, d] with lse [rows] in the same row order
    lse_rows = lambda t: t.permute(0, 2, 1).contiguous().reshape(rows)  # noqa: E731
    o_m, l_m = ra.merge(o_keep.reshape(rows, 128), lse_rows(l_keep), o_b.reshape(rows, 128),
                        lse_rows(l_b))
    ra.check_status()
    assert torch.equal(o_f.reshape(rows, 128), o_m)
    assert torch.equal(lse_rows(l_f), l_m)
    assert torch.equal(out_f, o_f.to(torch.bfloat16))
    # and the fold is the attention over both key blocks
    qc, kc1, vc1, kc2, vc2 = (t.cpu() for t in (q, k1, v1, k2, v2))
    s = 1.0 / 128 ** 0.5
    oa, la = oracle.block_attention(qc, kc1, vc1, s, KIND[mask_a])
    ob, lb = oracle.block_attention(qc, kc2, vc2, s, KIND[mask_b])
    o_ref, l_ref = oracle.merge(oa, la.transpose(0, 2, 1), ob, lb.transpose(0, 2, 1))
    compare_partial(o_f, l_f, o_ref, l_ref.transpose(0, 2, 1), "fold")


def test_strict_one_row_block_is_empty(ra):
    """l = 1 under the strict mask: the only row has no key."""
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = (t.cuda() for t in make_inputs(1, 2, 2, 1, 64, seed=33))
    o, l_, out = visit(ra, q, k, v, 2)
    assert torch.all(o == 0) and torch.all(torch.isneginf(l_)) and torch.all(out == 0)


# (layout, world, causal, B, Hq, Hkv, L, d)
RING_CASES = [
    ("contiguous", 4, True, 1, 4, 2, 1536, 128),
    ("zigzag", 4, True, 1, 4, 2, 1536, 128),
    ("striped", 4, True, 1, 4, 2, 1536, 128),
    ("zigzag", 3, True, 2, 2, 1, 1200, 64),       # chunks of 200 rows
    ("striped", 3, False, 1, 2, 2, 768, 128),
    ("zigzag", 2, False, 1, 2, 2, 1024, 128),
    ("contiguous", 1, True, 1, 2, 2, 640, 128),
    ("striped", 8, True, 1, 2, 1, 2048, 128),
]


@pytest.mark.parametrize("layout,world,causal,B,Hq,Hkv,L,d", RING_CASES)
def test_emulated_ring_matches_oracle(ra, layout, world, causal, B, Hq, Hkv, L, d):
    """Every host's visits and folds of the multi-process ring, run on one
    device with the CUDA visit, give exact attention over the sequence."""
    from ring_attention_ordered_b200 import ring
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, L, d, seed=L + world)
    out, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), world, causal,
                                            layout=layout)
    ra.check_status()
    o_ref, l_ref = oracle.attention(q, k, v, causal, 1.0 / d ** 0.5)
    compare(out, lse, o_ref, l_ref, f"{layout} N={world} causal={causal}")


def test_emulated_zigzag_ring_on_the_l8k_workload(ra):
    """The 8K-token causal workload (B 2, 8 heads, d 128) as a zigzag ring of
    4 hosts: sampled rows and every chunk boundary against the oracle."""
    from ring_attention_ordered_b200 import ring
    from ring_attention_ordered_b200.inputs import WORKLOADS, sample_rows, workload_inputs
    w = WORKLOADS["l8k_h8_causal"]
    q, k, v = workload_inputs(w)
    out, lse = ring.ring_attention_emulated(q.cuda(), k.cuda(), v.cuda(), w.n_ring, w.causal,
                                            w.scale, "zigzag")
    ra.check_status()
    c = w.L // (2 * w.n_ring)
    edges = sorted({r for g in range(2 * w.n_ring + 1) for r in (g * c - 1, g * c)
                    if 0 <= r < w.L})
    bhr = np.concatenate([sample_rows(w, 1024),
                          np.array([[b, h, r] for b in range(w.B) for h in (0, w.Hq - 1)
                                    for r in edges], dtype=np.int64)])
    o_ref, l_ref = oracle.attention_rows(q, k, v, w.causal, w.scale, bhr)
    b, h, r = (torch.from_numpy(bhr[:, i]).cuda() for i in range(3))
    compare(out[b, r, h, :], lse[b, h, r], o_ref, l_ref, "l8k zigzag")


# ------------------------------------------------------------------ backward

def fwd_stats_bf16(q, k, v, causal, scale):
    """Forward output (rounded to bf16) and lse of the oracle, as the inputs a
    backward visit takes."""
    o, l_ = oracle.attention(q, k, v, causal, scale)
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(l_).float()


@pytest.mark.parametrize("mask", [0, 1, 2])
@pytest.mark.parametrize("B,Hq,Hkv,l,d", [(1, 2, 2, 256, 128), (2, 4, 2, 200, 64),
                                          (1, 3, 1, 384, 128)])
def test_bwd_visit_matches_oracle(ra, B, Hq, Hkv, l, d, mask):
    """Both halves of one backward visit against block_attention_bwd, on the
    oracle's own forward output and lse; the accumulators start from values
    already there (fold) and dq is the rounding of the new dq_acc."""
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    from parity import compare_grad
    q, k, v = make_inputs(B, Hq, Hkv, l, d, seed=200 + l + mask)
    _, k2, v2 = make_inputs(B, Hq, Hkv, l, d, seed=300 + l + mask)   # another K/V block
    do = make_grad_output(B, l, Hq, d, seed=200 + l)
    scale = 1.0 / d ** 0.5
    out, lse = fwd_stats_bf16(q, k, v, True, scale)
    g = torch.Generator().manual_seed(5)
    dq0 = torch.randn(q.shape, generator=g)
    dk0, dv0 = torch.randn(k.shape, generator=g), torch.randn(k.shape, generator=g)
    dq_acc, dk_acc, dv_acc = dq0.cuda(), dk0.cuda(), dv0.cuda()
    dq = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(B * Hq * l * 4, dtype=torch.uint8, device="cuda")
    qd, kd, vd, od, dod, ld = (t.cuda() for t in (q, k2, v2, out, do, lse))
    ra.bwd_visit(qd, kd, vd, od, dod, ld, ws, mask, 1, dq_acc=dq_acc, fold_q=True, scale=scale,
                 dq=dq)
    ra.bwd_visit(qd, kd, vd, od, dod, ld, ws, mask, 2, dk_acc=dk_acc, dv_acc=dv_acc, fold_kv=True,
                 scale=scale)
    ra.check_status()
    pq, pk, pv = oracle.block_attention_bwd(q, k2, v2, out, do, lse, scale, KIND[mask])
    what = f"{(B, Hq, Hkv, l, d, mask)}"
    compare_grad(dq_acc.cpu() - dq0, pq, what + " dq")
    compare_grad(dk_acc.cpu() - dk0, pk, what + " dk")
    compare_grad(dv_acc.cpu() - dv0, pv, what + " dv")
    assert torch.equal(dq, dq_acc.to(torch.bfloat16))
    # without fold the accumulators are overwritten, whatever they held
    dq_acc2 = torch.full_like(dq_acc, float("nan"))
    ra.bwd_visit(qd, kd, vd, od, dod, ld, ws, mask, 3, dq_acc=dq_acc2,
                 dk_acc=torch.full_like(dk_acc, float("nan")),
                 dv_acc=torch.full_like(dv_acc, float("nan")), scale=scale)
    ra.check_status()
    compare_grad(dq_acc2.cpu(), pq, what + " dq (write)")


def test_round_bf16_is_round_to_nearest_even(ra):
    g = torch.Generator().manual_seed(6)
    x = torch.randn(1 << 16, generator=g) * 10.0
    x[:8] = torch.tensor([float("inf"), -float("inf"), 0.0, -0.0, 1e-40, 3.0e38, 1.00390625,
                          1.01171875])
    y = ra.round_bf16(x.cuda())
    ra.check_status()
    assert torch.equal(y.cpu().view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


# (layout, world, causal, B, Hq, Hkv, L, d)
RING_BWD_CASES = [
    ("contiguous", 4, True, 1, 4, 2, 1024, 128),
    ("zigzag", 4, True, 1, 4, 2, 1024, 128),
    ("striped", 4, True, 1, 4, 2, 1024, 128),
    ("zigzag", 3, False, 2, 2, 1, 1200, 64),
    ("contiguous", 1, True, 1, 2, 2, 384, 128),
    ("striped", 2, False, 1, 2, 2, 512, 128),
]


@pytest.mark.parametrize("layout,world,causal,B,Hq,Hkv,L,d", RING_BWD_CASES)
def test_emulated_ring_bwd_matches_oracle(ra, layout, world, causal, B, Hq, Hkv, L, d):
    """Every host's backward visits with the travelling dK, dV accumulators,
    on one device, against the definition's gradients."""
    from parity import compare_grad
    from ring_attention_ordered_b200 import ring
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, L, d, seed=L + 7 * world)
    do = make_grad_output(B, L, Hq, d, seed=L + 7 * world)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = ring.ring_attention_emulated(qd, kd, vd, world, causal, layout=layout)
    got = ring.ring_attention_bwd_emulated(qd, kd, vd, out, dod, lse, world, causal,
                                           layout=layout)
    ra.check_status()
    want = oracle.attention_bwd(q, k, v, do, causal, 1.0 / d ** 0.5)
    for g_, w_, n in zip(got, want, "qkv"):
        compare_grad(g_, w_, f"{layout} N={world} causal={causal} d{n}")
