"""GPU parity of ring_attn_merge (through the C ABI) against the fp64 oracle
merge, including the empty-partial and NaN rules, in-place use and bitwise
symmetry."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


def partials(rows, d, seed):
    g = torch.Generator().manual_seed(seed)
    o_a = torch.randn(rows, d, generator=g)
    o_b = torch.randn(rows, d, generator=g)
    l_a = torch.randn(rows, generator=g) * 20
    l_b = torch.randn(rows, generator=g) * 20
    if rows >= 16:
        l_a[3::11] = -float("inf")          # empty partial on side a
        o_a[3::11] = float("nan")           # whose o is garbage
        l_b[5::13] = -float("inf")
        l_a[7] = l_b[7] = -float("inf")     # both empty
        l_b[9] = float("nan")               # NaN propagates
        l_a[10] = l_b[10] + 0.0             # equal weights
    return o_a, l_a, o_b, l_b


def check(o, l_, o_a, l_a, o_b, l_b):
    ro, rl = oracle.merge(o_a.double().numpy(), l_a.double().numpy(),
                          o_b.double().numpy(), l_b.double().numpy())
    o = o.cpu().double().numpy()
    l_ = l_.cpu().double().numpy()
    nan_rows = np.isnan(rl)
    assert np.array_equal(np.isnan(l_), nan_rows)
    assert np.all(np.isnan(o[nan_rows]))
    ok = ~nan_rows
    np.testing.assert_array_equal(np.isneginf(l_[ok]), np.isneginf(rl[ok]))
    fin = ok & np.isfinite(rl)
    np.testing.assert_allclose(l_[fin], rl[fin], rtol=1e-6, atol=1e-5)
    np.testing.assert_allclose(o[ok], ro[ok], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("rows,d", [(1, 4), (37, 64), (1000, 128), (4099, 256), (513, 12)])
def test_merge_matches_oracle(ra, rows, d):
    o_a, l_a, o_b, l_b = partials(rows, d, seed=rows + d)
    o, l_ = ra.merge(o_a.cuda(), l_a.cuda(), o_b.cuda(), l_b.cuda())
    torch.cuda.synchronize()
    check(o, l_, o_a, l_a, o_b, l_b)


def test_merge_empty_side_is_exact_and_symmetric(ra):
    o_a, l_a, o_b, l_b = partials(2048, 128, seed=5)
    A = [t.cuda() for t in (o_a, l_a)]
    Bt = [t.cuda() for t in (o_b, l_b)]
    o1, l1 = ra.merge(A[0], A[1], Bt[0], Bt[1])
    o2, l2 = ra.merge(Bt[0], Bt[1], A[0], A[1])
    torch.cuda.synchronize()
    assert torch.equal(o1.nan_to_num(7.0), o2.nan_to_num(7.0))
    assert torch.equal(l1.nan_to_num(7.0), l2.nan_to_num(7.0))
    empty_a = torch.isneginf(l_a) & torch.isfinite(l_b)
    assert torch.equal(o1.cpu()[empty_a], o_b[empty_a])
    assert torch.equal(l1.cpu()[empty_a], l_b[empty_a])


def test_merge_in_place(ra):
    o_a, l_a, o_b, l_b = partials(3000, 128, seed=6)
    A0, A1 = o_a.cuda(), l_a.cuda()
    ra.merge(A0, A1, o_b.cuda(), l_b.cuda(), out=A0, lse_out=A1)
    torch.cuda.synchronize()
    check(A0, A1, o_a, l_a, o_b, l_b)


def test_merge_folds_ring_partials(ra):
    """Folding per-visit partials in ring order with the GPU merge gives full
    attention (oracle partials over key blocks, GPU folds)."""
    rng = np.random.default_rng(8)
    L, d, n = 256, 64, 4
    q, k, v = (rng.standard_normal((1, L, 1, d)) for _ in range(3))
    o_ref, l_ref = oracle.attention(q, k, v, False, 0.125)
    lb = L // n
    acc_o = torch.zeros(L, d, device="cuda")
    acc_l = torch.full((L,), -float("inf"), device="cuda")
    for i in range(n):
        rows = slice(i * lb, (i + 1) * lb)
        for _, j, _ in oracle.ring_visits(i, n, False):
            s = 0.125 * q[0, rows, 0] @ k[0, j * lb:(j + 1) * lb, 0].T
            m = s.max(axis=1)
            e = np.exp(s - m[:, None])
            po = (e @ v[0, j * lb:(j + 1) * lb, 0]) / e.sum(axis=1)[:, None]
            pl = m + np.log(e.sum(axis=1))
            ao, al = acc_o[rows].contiguous(), acc_l[rows].contiguous()
            no, nl = ra.merge(ao, al, torch.tensor(po, dtype=torch.float32, device="cuda"),
                              torch.tensor(pl, dtype=torch.float32, device="cuda"))
            acc_o[rows], acc_l[rows] = no, nl
    torch.cuda.synchronize()
    np.testing.assert_allclose(acc_o.cpu().numpy(), o_ref[0, :, 0], rtol=0, atol=1e-5)
    np.testing.assert_allclose(acc_l.cpu().numpy(), l_ref[0, 0], rtol=0, atol=1e-5)


def test_merge_zero_rows_is_noop(ra):
    from ring_attention_ordered_b200 import _lib
    assert _lib.ring_attn_merge(0, 0, 0, 0, 0, 0, 0, 128, 0) == _lib.RA_OK
