"""Pins of the fp64 backward oracle (oracle/attn_bwd_fp64.py) against things
other than itself: torch autograd through fp64 scaled_dot_product_attention
(a library routine), central finite differences of the pinned forward
oracle, closed forms and invariants; and planted mistakes that each fail at
least one pin."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import attn_bwd_fp64 as ob
from oracle import attn_fp64 as oa


def rand(rng, *shape):
    return rng.standard_normal(shape)


def problem(seed, B=2, L=13, Hq=4, Hkv=2, d=6):
    rng = np.random.default_rng(seed)
    return (rand(rng, B, L, Hq, d), rand(rng, B, L, Hkv, d), rand(rng, B, L, Hkv, d),
            rand(rng, B, L, Hq, d))


def pin_autograd(bwd, causal=True):
    """torch autograd of fp64 SDPA (GQA grouping included)."""
    q, k, v, do = problem(1)
    scale = 0.41
    dq, dk, dv = bwd(q, k, v, do, causal, scale)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).requires_grad_() for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal,
                                                         scale=scale, enable_gqa=True)
    o.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    for got, t in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(got, t.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def pin_finite_differences(bwd, causal=True):
    """Central differences of sum(O * dO), O from the (separately pinned)
    forward oracle, for every input element of a tiny problem."""
    q, k, v, do = problem(2, B=1, L=5, Hq=2, Hkv=1, d=3)
    scale = 0.9
    grads = bwd(q, k, v, do, causal, scale)

    def loss(qq, kk, vv):
        return float((oa.attention(qq, kk, vv, causal, scale)[0] * do).sum())

    h = 1e-6
    for which, x in enumerate((q, k, v)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][idx] += h
            up = loss(*args)
            args[which][idx] -= 2 * h
            num[idx] = (up - loss(*args)) / (2 * h)
        np.testing.assert_allclose(grads[which], num, rtol=0, atol=1e-7)


def pin_invariants(bwd):
    """Every row of dS sums to zero, so the key gradients of each K/V head
    sum to zero; dO = 0 gives zero gradients; when every key carries the same
    value row, O does not depend on Q or K (dQ = dK = 0) and dV sums over
    keys to the sum of dO over the group's rows."""
    q, k, v, do = problem(3)
    for causal in (False, True):
        _, dk, _ = bwd(q, k, v, do, causal, 0.5)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, rtol=0, atol=1e-12)
        zq, zk, zv = bwd(q, k, v, np.zeros_like(do), causal, 0.5)
        assert not zq.any() and not zk.any() and not zv.any()
        cv = np.broadcast_to(v[:, :1], v.shape).copy()
        dq, dk, dv = bwd(q, k, cv, do, causal, 0.5)
        np.testing.assert_allclose(dq, 0.0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk, 0.0, rtol=0, atol=1e-12)
        g = q.shape[2] // k.shape[2]
        want = do.reshape(do.shape[0], do.shape[1], k.shape[2], g, do.shape[3]).sum(axis=(1, 3))
        np.testing.assert_allclose(dv.sum(axis=1), want, rtol=0, atol=1e-12)


def pin_causal_last_key(bwd):
    """Under causal masking the last key is seen only by the last query row,
    with weight A = exp(s - lse) of that row: dV[L-1] = A dO[L-1] per head."""
    q, k, v, do = problem(4, B=1, Hq=2, Hkv=2)
    scale = 0.7
    _, _, dv = bwd(q, k, v, do, True, scale)
    _, lse = oa.brute_attention(q, k, v, True, scale)
    L = q.shape[1]
    for h in range(2):
        a = np.exp(scale * q[0, L - 1, h] @ k[0, L - 1, h] - lse[0, h, L - 1])
        np.testing.assert_allclose(dv[0, L - 1, h], a * do[0, L - 1, h], rtol=1e-12, atol=1e-14)


BWD_PINS = [pin_autograd, pin_finite_differences, pin_invariants, pin_causal_last_key]


@pytest.mark.parametrize("pin", BWD_PINS)
def test_bwd_pins(pin):
    pin(oracle.attention_bwd)


def test_bwd_non_causal_autograd():
    pin_autograd(oracle.attention_bwd, causal=False)
    pin_finite_differences(oracle.attention_bwd, causal=False)


@pytest.mark.parametrize("causal", [False, True])
def test_row_functions_match_the_full_gradient(causal):
    q, k, v, do = problem(5, B=2, L=40, Hq=6, Hkv=2, d=8)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, 0.3)
    rng = np.random.default_rng(0)
    bhr = np.stack([rng.integers(0, 2, 30), rng.integers(0, 6, 30), rng.integers(0, 40, 30)], 1)
    np.testing.assert_allclose(oracle.attention_bwd_dq_rows(q, k, v, do, causal, 0.3, bhr),
                               dq[bhr[:, 0], bhr[:, 2], bhr[:, 1]], rtol=0, atol=1e-12)
    bhc = np.stack([rng.integers(0, 2, 30), rng.integers(0, 2, 30), rng.integers(0, 40, 30)], 1)
    gk, gv = oracle.attention_bwd_kv_rows(q, k, v, do, causal, 0.3, bhc, row_block=7)
    np.testing.assert_allclose(gk, dk[bhc[:, 0], bhc[:, 2], bhc[:, 1]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(gv, dv[bhc[:, 0], bhc[:, 2], bhc[:, 1]], rtol=0, atol=1e-12)


def test_bf16_torch_inputs_are_accepted():
    g = torch.Generator().manual_seed(9)
    q, k, v, do = (torch.randn(s, generator=g).to(torch.bfloat16)
                   for s in ((1, 9, 2, 4), (1, 9, 1, 4), (1, 9, 1, 4), (1, 9, 2, 4)))
    a = oracle.attention_bwd(q, k, v, do, True, 0.5)
    b = oracle.attention_bwd(*(x.float().numpy() for x in (q, k, v, do)), True, 0.5)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


# --------------------------------------------------------------------------
# planted mistakes
# --------------------------------------------------------------------------

def _fails(pin, fn):
    try:
        with np.errstate(all="ignore"):
            pin(fn)
    except (AssertionError, ValueError, FloatingPointError):
        return True
    return False


def _mutant(mistake):
    def bwd(q, k, v, dout, causal, scale):
        q, k, v, do = (oa._f64(x) for x in (q, k, v, dout))
        B, L, Hq, Hkv, d, g = oa._shapes(q, k, v)
        dq = np.zeros((B, L, Hq, d))
        dk = np.zeros((B, L, Hkv, d))
        dv = np.zeros((B, L, Hkv, d))
        for b in range(B):
            for h in range(Hq):
                kh = h // g
                s = scale * (q[b, :, h] @ k[b, :, kh].T)
                if causal and mistake != "mask_dropped":
                    s[np.triu_indices(L, 1)] = -np.inf
                e = np.exp(s - s.max(axis=1, keepdims=True))
                a = e / e.sum(axis=1, keepdims=True)
                da = do[b, :, h] @ v[b, :, kh].T
                if mistake == "no_row_term":
                    ds = a * da
                elif mistake == "row_term_of_da":
                    ds = a * (da - da.sum(axis=1, keepdims=True))
                else:
                    ds = a * (da - (a * da).sum(axis=1, keepdims=True))
                if mistake == "dv_untransposed":
                    dv[b, :, kh] += a @ do[b, :, h]
                else:
                    dv[b, :, kh] += a.T @ do[b, :, h]
                dq[b, :, h] = (1.0 if mistake == "dq_no_scale" else scale) * (ds @ k[b, :, kh])
                if mistake == "gqa_last_head_only":
                    dk[b, :, kh] = scale * (ds.T @ q[b, :, h])
                else:
                    dk[b, :, kh] += scale * (ds.T @ q[b, :, h])
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("mistake", ["mask_dropped", "no_row_term", "row_term_of_da",
                                     "dv_untransposed", "dq_no_scale", "gqa_last_head_only"])
def test_planted_bwd_mistake_is_caught(mistake):
    assert any(_fails(pin, _mutant(mistake)) for pin in BWD_PINS), mistake


def test_clean_bwd_mutant_template_passes():
    for pin in BWD_PINS:
        pin(_mutant(None))
    assert ob.attention_bwd is oracle.attention_bwd


# --------------------------------------------------------------------------
# block_attention_bwd: one ring visit's share of the gradients
# --------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_blocks", [1, 2, 4])
def test_block_bwd_parts_sum_to_the_gradient(causal, n_blocks):
    """With the forward oracle's own output and lse, the parts of every
    (query block, key block) pair the mask allows -- diagonal blocks
    "masked", earlier blocks "full" -- add up to attention_bwd."""
    q, k, v, do = problem(6, B=2, L=24, Hq=4, Hkv=2, d=5)
    scale = 0.45
    out, lse = oa.attention(q, k, v, causal, scale)
    want = oracle.attention_bwd(q, k, v, do, causal, scale)
    lb = 24 // n_blocks
    got = [np.zeros_like(x) for x in (q, k, v)]
    for i in range(n_blocks):
        rq = slice(i * lb, (i + 1) * lb)
        for j in range(n_blocks):
            if causal and j > i:
                continue
            rk = slice(j * lb, (j + 1) * lb)
            kind = "masked" if (causal and i == j) else "full"
            pq, pk, pv = oracle.block_attention_bwd(q[:, rq], k[:, rk], v[:, rk], out[:, rq],
                                                    do[:, rq], lse[:, :, rq], scale, kind)
            got[0][:, rq] += pq
            got[1][:, rk] += pk
            got[2][:, rk] += pv
    for g_, w_ in zip(got, want):
        np.testing.assert_allclose(g_, w_, rtol=0, atol=1e-12)


def test_block_bwd_strict_is_the_shifted_masked_visit():
    """Keys c < r: row 0 receives nothing and key L-1 gives nothing; the
    strict visit equals the masked visit minus the diagonal pairs, checked
    by adding the diagonal's share, formed from the definition one pair at a
    time with math.fsum."""
    import math
    q, k, v, do = problem(7, B=1, L=6, Hq=2, Hkv=1, d=3)
    scale = 0.8
    out, lse = oa.attention(q, k, v, True, scale)
    sq, sk, sv = oracle.block_attention_bwd(q, k, v, out, do, lse, scale, "strict")
    mq, mk, mv = oracle.block_attention_bwd(q, k, v, out, do, lse, scale, "masked")
    assert np.all(sq[:, 0] == 0.0)
    dq_d, dk_d, dv_d = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(2):
        for r in range(6):
            a = math.exp(scale * math.fsum(q[0, r, h] * k[0, r, 0]) - lse[0, h, r])
            da = math.fsum(do[0, r, h] * v[0, r, 0])
            rt = math.fsum(do[0, r, h] * out[0, r, h])
            ds = a * (da - rt)
            dv_d[0, r, 0] += a * do[0, r, h]
            dq_d[0, r, h] += scale * ds * k[0, r, 0]
            dk_d[0, r, 0] += scale * ds * q[0, r, h]
    for s_, m_, d_ in ((sq, mq, dq_d), (sk, mk, dk_d), (sv, mv, dv_d)):
        np.testing.assert_allclose(s_ + d_, m_, rtol=0, atol=1e-12)
