"""Pins of the fp64 oracle against things other than itself.

Each pin is a function taking the implementation under test, so that the
mutation tests at the end can plant a plausible mistake in a copy of the
oracle and show that some pin fails.  All of this runs on the CPU.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attn_fp64 as oa

RNG = np.random.default_rng(1234)


def rand(*shape, rng=RNG):
    return rng.standard_normal(shape)


def bf16_values(*shape, seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).float().numpy()


# --------------------------------------------------------------------------
# pins, parameterised by the implementation
# --------------------------------------------------------------------------

def pin_brute(attn, B=2, L=9, Hq=4, Hkv=2, d=5, causal=True, seed=0):
    """Brute-force triple loop with exactly rounded sums on a tiny input."""
    rng = np.random.default_rng(seed)
    q, k, v = rand(B, L, Hq, d, rng=rng), rand(B, L, Hkv, d, rng=rng), rand(B, L, Hkv, d, rng=rng)
    scale = 0.7
    o, l_ = attn(q, k, v, causal, scale)
    ob, lb = oa.brute_attention(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_, lb, rtol=0, atol=1e-12)


def pin_sdpa(attn, B=2, L=37, Hq=6, Hkv=3, d=16, causal=True, seed=1):
    """torch's scaled_dot_product_attention in float64 on the CPU (a library
    routine for the same definition), including its GQA head grouping."""
    rng = np.random.default_rng(seed)
    q, k, v = rand(B, L, Hq, d, rng=rng), rand(B, L, Hkv, d, rng=rng), rand(B, L, Hkv, d, rng=rng)
    scale = 1.0 / math.sqrt(d)
    o, _ = attn(q, k, v, causal, scale)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(
        tq, tk, tv, is_causal=causal, scale=scale, enable_gqa=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def pin_causal_row0(attn, L=16, d=8):
    """Causal row 0 sees key 0 only: O[0] = v_0 and lse[0] = scale * q_0.k_0."""
    q, k, v = rand(1, L, 2, d), rand(1, L, 1, d), rand(1, L, 1, d)
    scale = 0.3
    o, l_ = attn(q, k, v, True, scale)
    for h in range(2):
        np.testing.assert_array_equal(o[0, 0, h], v[0, 0, 0])
        assert abs(l_[0, h, 0] - scale * float(q[0, 0, h] @ k[0, 0, 0])) < 1e-14


def pin_zero_query(attn, L=20, d=6, causal=True):
    """Q = 0 makes every allowed key equally likely: O[r] is the mean of the
    allowed values and lse[r] = ln(number of allowed keys)."""
    q = np.zeros((1, L, 1, d))
    k, v = rand(1, L, 1, d), rand(1, L, 1, d)
    o, l_ = attn(q, k, v, causal, 1.0)
    for r in range(L):
        n = r + 1 if causal else L
        np.testing.assert_allclose(o[0, r, 0], v[0, :n, 0].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(l_[0, 0, r] - math.log(n)) < 1e-14


def pin_constant_values(attn, L=24, d=7, causal=False):
    """Constant V reproduces V (the weights of a row sum to one)."""
    q, k = rand(1, L, 2, d), rand(1, L, 2, d)
    c = rand(d)
    v = np.broadcast_to(c, (1, L, 2, d)).copy()
    o, _ = attn(q, k, v, causal, 0.9)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-13)


def pin_key_shift(attn, L=18, d=5, causal=True):
    """Adding one vector c to every key leaves O unchanged and moves lse[r]
    by scale * q_r . c (softmax is invariant to a per-row constant)."""
    q, k, v = rand(1, L, 1, d), rand(1, L, 1, d), rand(1, L, 1, d)
    c = rand(d)
    scale = 0.8
    o1, l1 = attn(q, k, v, causal, scale)
    o2, l2 = attn(q, k + c, v, causal, scale)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2[0, 0] - l1[0, 0], scale * (q[0, :, 0] @ c), rtol=0, atol=1e-12)


def pin_one_hot_peak(attn, L=12, d=4):
    """A key whose score dominates by a huge margin takes all the weight: O
    equals that key's value and lse its score (textbook limit of softmax)."""
    q = np.zeros((1, L, 1, d))
    q[0, :, 0, 0] = 1.0
    k = np.zeros((1, L, 1, d))
    k[0, 5, 0, 0] = 2000.0
    v = rand(1, L, 1, d)
    o, l_ = attn(q, k, v, False, 1.0)
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, 5, 0], (L, d)), rtol=0, atol=1e-300)
    np.testing.assert_allclose(l_[0, 0], 2000.0, rtol=0, atol=1e-12)


ALL_ATTENTION_PINS = [pin_brute, pin_sdpa, pin_causal_row0, pin_zero_query,
                      pin_constant_values, pin_key_shift, pin_one_hot_peak]


def pin_ring_equals_direct(ring, attn, n_ring, causal, L=24, Hq=4, Hkv=2, d=6, seed=3):
    """The ring-ordered blockwise result equals full attention: the pages
    call the method exact, not an approximation."""
    rng = np.random.default_rng(seed)
    q, k, v = rand(2, L, Hq, d, rng=rng), rand(2, L, Hkv, d, rng=rng), rand(2, L, Hkv, d, rng=rng)
    scale = 0.6
    o1, l1 = ring(q, k, v, n_ring, causal, scale)
    o2, l2 = attn(q, k, v, causal, scale)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def pin_ring_order_golden(order, golden_dir):
    rows = np.loadtxt(os.path.join(golden_dir, "ring_order_n4.txt"), dtype=int, comments="#")
    for row in rows:
        t, blocks = int(row[0]), [int(x) for x in row[1:]]
        assert [order(i, 4)[t] for i in range(4)] == blocks


def pin_merge_split_keys(merge, attn, L=30, d=5, cut=11, seed=5):
    """Attention over keys A u B equals the merge of attention over A and
    attention over B (disjoint, non-empty), in either order."""
    rng = np.random.default_rng(seed)
    q, k, v = rand(1, L, 1, d, rng=rng), rand(1, L, 1, d, rng=rng), rand(1, L, 1, d, rng=rng)
    scale = 0.9
    o, l_ = attn(q, k, v, False, scale)
    # attention of all L queries against the first `cut` keys and the rest:
    # pad q so the query count matches the key count of each part
    def part(lo, hi):
        rows_o = np.empty((L, d))
        rows_l = np.empty(L)
        for r in range(L):
            s = scale * (k[0, lo:hi, 0] @ q[0, r, 0])
            m = s.max()
            e = np.exp(s - m)
            rows_o[r] = (e @ v[0, lo:hi, 0]) / e.sum()
            rows_l[r] = m + math.log(e.sum())
        return rows_o, rows_l
    oa_, la_ = part(0, cut)
    ob_, lb_ = part(cut, L)
    om, lm = merge(oa_, la_, ob_, lb_)
    np.testing.assert_allclose(om, o[0, :, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lm, l_[0, 0], rtol=0, atol=1e-12)


def pin_merge_closed_forms(merge):
    """merge(x, x) = (o, lse + ln 2); an empty partial is the identity; two
    empty partials stay empty; weights follow exp(lse)."""
    o = rand(7, 4)
    l_ = rand(7)
    om, lm = merge(o, l_, o, l_)
    np.testing.assert_allclose(om, o, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lm, l_ + math.log(2.0), rtol=0, atol=1e-14)
    empty_o = np.full((7, 4), np.nan)
    empty_l = np.full(7, -np.inf)
    om, lm = merge(empty_o, empty_l, o, l_)
    np.testing.assert_array_equal(om, o)
    np.testing.assert_array_equal(lm, l_)
    om, lm = merge(empty_o, empty_l, empty_o, empty_l)
    np.testing.assert_array_equal(om, np.zeros_like(o))
    assert np.all(lm == -np.inf)
    # two partials with lse 0 and ln 3: weights 1/4 and 3/4
    a, b = rand(3), rand(3)
    om, lm = merge(a[None], np.array([0.0]), b[None], np.array([math.log(3.0)]))
    np.testing.assert_allclose(om[0], 0.25 * a + 0.75 * b, rtol=0, atol=1e-15)
    assert abs(lm[0] - math.log(4.0)) < 1e-15


# --------------------------------------------------------------------------
# the oracle against its pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("pin", ALL_ATTENTION_PINS, ids=lambda p: p.__name__)
def test_attention_pins(pin):
    pin(oracle.attention)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_brute_both_masks(causal):
    pin_brute(oracle.attention, causal=causal)
    pin_sdpa(oracle.attention, causal=causal)


def test_attention_rows_matches_full():
    q, k, v = rand(2, 40, 4, 8), rand(2, 40, 2, 8), rand(2, 40, 2, 8)
    for causal in (False, True):
        o, l_ = oracle.attention(q, k, v, causal, 0.5)
        bhr = np.array([[b, h, r] for b in range(2) for h in range(4) for r in range(0, 40, 3)])
        orow, lrow = oracle.attention_rows(q, k, v, causal, 0.5, bhr, row_block=5)
        # equal up to the summation order of the library matmul
        np.testing.assert_allclose(orow, o[bhr[:, 0], bhr[:, 2], bhr[:, 1]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lrow, l_[bhr[:, 0], bhr[:, 1], bhr[:, 2]], rtol=0, atol=1e-14)


def test_attention_rows_pins():
    def via_rows(q, k, v, causal, scale):
        B, L, Hq, d = q.shape
        bhr = np.array([[b, h, r] for b in range(B) for h in range(Hq) for r in range(L)])
        o, l_ = oracle.attention_rows(q, k, v, causal, scale, bhr, row_block=7)
        out = np.empty((B, L, Hq, d))
        lse = np.empty((B, Hq, L))
        out[bhr[:, 0], bhr[:, 2], bhr[:, 1]] = o
        lse[bhr[:, 0], bhr[:, 1], bhr[:, 2]] = l_
        return out, lse
    for pin in ALL_ATTENTION_PINS:
        pin(via_rows)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    q, k = rand(1, 15, 2, 4), rand(1, 15, 1, 4)
    p = oracle.attention_probs(q, k, causal, 1.1)
    np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=0, atol=1e-14)
    assert np.all(p >= 0)
    if causal:
        assert np.all(p[..., np.triu_indices(15, 1)[0], np.triu_indices(15, 1)[1]] == 0)
    # the weights reproduce the output
    v = rand(1, 15, 1, 4)
    o, _ = oracle.attention(q, k, v, causal, 1.1)
    np.testing.assert_allclose(o[0, :, 1], p[0, 1] @ v[0, :, 0], rtol=0, atol=1e-13)


def test_bf16_inputs_are_exact_in_fp64():
    x = bf16_values(3, 5, 2, 4)
    t = torch.from_numpy(x).to(torch.bfloat16)
    np.testing.assert_array_equal(oa._f64(t.float().numpy()), x.astype(np.float64))


@pytest.mark.parametrize("n_ring", [1, 2, 3, 4, 8, 12, 24])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_equals_direct(n_ring, causal):
    pin_ring_equals_direct(oracle.ring_attention, oracle.attention, n_ring, causal)
    pin_ring_equals_direct(oracle.ring_attention_merged, oracle.attention, n_ring, causal)


def test_ring_n16_bf16_inputs():
    q = bf16_values(1, 64, 2, 8, seed=1)
    k = bf16_values(1, 64, 1, 8, seed=2)
    v = bf16_values(1, 64, 1, 8, seed=3)
    for causal in (False, True):
        o1, l1 = oracle.ring_attention(q, k, v, 16, causal, 8 ** -0.5)
        o2, l2 = oracle.attention(q, k, v, causal, 8 ** -0.5)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_ring_n1_is_plain_attention():
    q, k, v = rand(1, 10, 1, 3), rand(1, 10, 1, 3), rand(1, 10, 1, 3)
    for causal in (False, True):
        o1, l1 = oracle.ring_attention(q, k, v, 1, causal, 1.0)
        o2, l2 = oracle.attention(q, k, v, causal, 1.0)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_ring_order_worked_example(golden_dir):
    pin_ring_order_golden(oracle.ring_order, golden_dir)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 16])
def test_ring_order_is_a_rotation(n):
    for i in range(n):
        order = oracle.ring_order(i, n)
        assert sorted(order) == list(range(n))
        assert order[0] == i
        # at step t host i holds what host i-1 held at step t-1
        for t in range(1, n):
            assert order[t] == oracle.ring_order((i - 1) % n, n)[t - 1]


@pytest.mark.parametrize("n", [1, 2, 3, 4, 8, 16])
def test_causal_visits(n):
    for i in range(n):
        visits = oracle.ring_visits(i, n, True)
        # the own (diagonal) block first, then the earlier blocks, latest first
        assert [j for _, j, _ in visits] == list(range(i, -1, -1))
        assert visits[0][2] == "masked"
        assert all(kind == "full" for _, _, kind in visits[1:])
        assert [t for t, _, _ in visits] == list(range(i + 1))
    computed, masked, skipped = oracle.causal_pair_counts(n)
    assert computed == n * (n + 1) // 2
    assert masked == n
    assert skipped == n * (n - 1) // 2


def test_causal_waste_tends_to_half():
    # the pages put the causal waste of the plain ring at 50%: the skipped
    # share N(N-1)/2 / N^2 tends to one half as N grows
    shares = [oracle.causal_pair_counts(n)[2] / n ** 2 for n in (2, 8, 64, 512)]
    assert shares == sorted(shares)
    assert abs(shares[-1] - 0.5) < 1e-3


def test_kv_bytes_worked_example(golden_dir):
    row = np.loadtxt(os.path.join(golden_dir, "kv_block_bytes.txt"), dtype=np.int64, comments="#")
    assert oracle.kv_bytes_per_ring_step(*[int(x) for x in row[:4]]) == int(row[4])
    assert int(row[4]) == 256 * 2 ** 20


def test_merge_split_keys():
    pin_merge_split_keys(oracle.merge, oracle.attention)
    pin_merge_split_keys(lambda oa_, la, ob, lb: oracle.merge(ob, lb, oa_, la), oracle.attention)


def test_merge_closed_forms():
    pin_merge_closed_forms(oracle.merge)


def test_merge_bitwise_commutative_and_associative():
    rng = np.random.default_rng(7)
    o = [rng.standard_normal((50, 8)) for _ in range(3)]
    l_ = [rng.standard_normal(50) * 30 for _ in range(3)]
    l_[1][::7] = -np.inf
    ab = oracle.merge(o[0], l_[0], o[1], l_[1])
    ba = oracle.merge(o[1], l_[1], o[0], l_[0])
    np.testing.assert_array_equal(ab[0], ba[0])
    np.testing.assert_array_equal(ab[1], ba[1])
    left = oracle.merge(*ab, o[2], l_[2])
    right = oracle.merge(o[0], l_[0], *oracle.merge(o[1], l_[1], o[2], l_[2]))
    np.testing.assert_allclose(left[0], right[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(left[1], right[1], rtol=1e-12, atol=0)


def test_merge_nan_propagates():
    o = np.ones((2, 3))
    om, lm = oracle.merge(o, np.array([np.nan, 0.0]), o, np.array([0.0, 0.0]))
    assert np.isnan(lm[0]) and np.all(np.isnan(om[0]))
    assert lm[1] == math.log(2.0)


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# --------------------------------------------------------------------------

def _fails(fn, *args):
    try:
        with np.errstate(all="ignore"):
            fn(*args)
    except (AssertionError, ValueError, FloatingPointError, IndexError):
        return True
    return False


def _mutant_attention(mistake):
    def attn(q, k, v, causal, scale):
        q, k, v = oa._f64(q), oa._f64(k), oa._f64(v)
        B, L, Hq, Hkv, d, g = oa._shapes(q, k, v)
        out = np.empty((B, L, Hq, d))
        lse = np.empty((B, Hq, L))
        for b in range(B):
            for h in range(Hq):
                kh = h % Hkv if mistake == "gqa_interleaved" else h // g
                kk = k[b, :, kh, :]
                s = (q[b, :, h, :] @ kk.T) * (scale if mistake != "no_scale" else 1.0)
                if mistake == "k_transposed":
                    s = s.T
                if causal:
                    off = 0 if mistake == "mask_off_by_one" else 1
                    s[np.triu_indices(L, off)] = -np.inf
                m = s.max(axis=1)
                e = np.exp(s - m[:, None])
                z = e.sum(axis=1)
                vals = v[b, :, kh, :]
                out[b, :, h, :] = (e @ vals) / (z[:, None] if mistake != "no_norm" else 1.0)
                lse[b, h] = (m + np.log(z)) if mistake != "lse_drops_max" else np.log(z)
        return out, lse
    return attn


@pytest.mark.parametrize("mistake", ["gqa_interleaved", "no_scale", "k_transposed",
                                     "mask_off_by_one", "no_norm", "lse_drops_max"])
def test_planted_attention_mistake_is_caught(mistake):
    mutant = _mutant_attention(mistake)
    assert any(_fails(pin, mutant) for pin in ALL_ATTENTION_PINS), mistake


def test_clean_mutant_template_passes():
    # the template with no mistake passes every pin, so the failures above
    # come from the planted mistakes alone
    for pin in ALL_ATTENTION_PINS:
        pin(_mutant_attention(None))


def _mutant_ring(mistake):
    def ring(q, k, v, n_ring, causal, scale):
        q, k, v = oa._f64(q), oa._f64(k), oa._f64(v)
        B, L, Hq, Hkv, d, g = oa._shapes(q, k, v)
        lb = L // n_ring
        out = np.empty((B, L, Hq, d))
        lse = np.empty((B, Hq, L))
        for b in range(B):
            for h in range(Hq):
                kh = h // g
                for i in range(n_ring):
                    qi = q[b, i * lb:(i + 1) * lb, h]
                    m = np.full(lb, -np.inf)
                    ls = np.zeros(lb)
                    o = np.zeros((lb, d))
                    visits = oa.ring_visits(i, n_ring, causal)
                    if mistake == "skip_diag_mask":
                        visits = [(t, j, "full") for t, j, _ in visits]
                    if mistake == "causal_keeps_later_blocks":
                        visits = [(t, j, "masked" if j == i and causal else "full")
                                  for t, j in enumerate(oa.ring_order(i, n_ring))]
                    for _, j, kind in visits:
                        s = oa._block_scores(qi, k[b, j * lb:(j + 1) * lb, kh], scale, kind)
                        m_new = np.maximum(m, s.max(axis=1))
                        alpha = np.exp(m - m_new) if mistake != "no_rescale" else np.ones(lb)
                        p = np.exp(s - m_new[:, None])
                        ls = alpha * ls + p.sum(axis=1)
                        o = alpha[:, None] * o + p @ v[b, j * lb:(j + 1) * lb, kh]
                        if mistake == "normalise_every_step":
                            o = o / ls[:, None]
                        m = m_new
                    out[b, i * lb:(i + 1) * lb, h] = o / ls[:, None]
                    lse[b, h, i * lb:(i + 1) * lb] = m + np.log(ls)
        return out, lse
    return ring


@pytest.mark.parametrize("mistake", ["skip_diag_mask", "causal_keeps_later_blocks",
                                     "no_rescale", "normalise_every_step"])
def test_planted_ring_mistake_is_caught(mistake):
    mutant = _mutant_ring(mistake)
    caught = any(_fails(pin_ring_equals_direct, mutant, oracle.attention, n, c)
                 for n in (2, 4) for c in (False, True))
    assert caught, mistake
    for n in (2, 4):
        for c in (False, True):
            pin_ring_equals_direct(_mutant_ring(None), oracle.attention, n, c)


def test_planted_ring_order_mistake_is_caught(golden_dir):
    assert _fails(pin_ring_order_golden, lambda i, n: [(i + t) % n for t in range(n)], golden_dir)


@pytest.mark.parametrize("mistake", ["sign", "no_max_shift_in_lse", "unweighted"])
def test_planted_merge_mistake_is_caught(mistake):
    def mutant(o_a, l_a, o_b, l_b):
        oa_, ob = np.asarray(o_a, float), np.asarray(o_b, float)
        mx = np.maximum(l_a, l_b)
        wa = np.exp(l_a - mx)
        wb = np.exp((mx - l_b) if mistake == "sign" else (l_b - mx))
        if mistake == "unweighted":
            wa = wb = np.ones_like(wa)
        den = wa + wb
        o = (wa[:, None] * oa_ + wb[:, None] * ob) / den[:, None]
        lse = np.log(den) if mistake == "no_max_shift_in_lse" else mx + np.log(den)
        return o, lse
    assert _fails(pin_merge_split_keys, mutant, oracle.attention) or _fails(pin_merge_closed_forms, mutant)


# --------------------------------------------------------------------------
# block_attention: one ring visit as a partial result
# --------------------------------------------------------------------------

def pin_block_full_and_masked(block):
    """"full" and "masked" visits are plain and causal attention of the
    block, checked against the exactly rounded brute force."""
    rng = np.random.default_rng(21)
    q, k, v = rand(2, 7, 4, 5, rng=rng), rand(2, 7, 2, 5, rng=rng), rand(2, 7, 2, 5, rng=rng)
    for kind, causal in (("full", False), ("masked", True)):
        o, l_ = block(q, k, v, 0.6, kind)
        ob, lb = oa.brute_attention(q, k, v, causal, 0.6)
        np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l_, lb, rtol=0, atol=1e-12)


def pin_block_strict_is_shifted_causal(block):
    """"strict" (keys c < r): row r of the block sees keys 0..r-1, which is
    row r-1 of causal attention of q[1:] against k[:-1], v[:-1] (brute
    force); row 0 has no key: o = 0, lse = -inf."""
    rng = np.random.default_rng(22)
    q, k, v = rand(1, 8, 2, 4, rng=rng), rand(1, 8, 1, 4, rng=rng), rand(1, 8, 1, 4, rng=rng)
    o, l_ = block(q, k, v, 0.8, "strict")
    ob, lb = oa.brute_attention(q[:, 1:], k[:, :-1], v[:, :-1], True, 0.8)
    np.testing.assert_allclose(o[:, 1:], ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l_[:, :, 1:], lb, rtol=0, atol=1e-12)
    assert np.all(o[:, 0] == 0.0) and np.all(l_[:, :, 0] == -np.inf)


def pin_block_unequal_lengths(block):
    """A "full" visit of 5 query rows against 11 keys: torch's fp64
    scaled_dot_product_attention (a library routine) with GQA grouping."""
    rng = np.random.default_rng(23)
    q, k, v = rand(1, 5, 4, 8, rng=rng), rand(1, 11, 2, 8, rng=rng), rand(1, 11, 2, 8, rng=rng)
    o, _ = block(q, k, v, 0.35, "full")
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=0.35,
                                                           enable_gqa=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


BLOCK_PINS = [pin_block_full_and_masked, pin_block_strict_is_shifted_causal,
              pin_block_unequal_lengths]


@pytest.mark.parametrize("pin", BLOCK_PINS)
def test_block_attention_pins(pin):
    pin(oracle.block_attention)


def _mutant_block(mistake):
    def block(q, k, v, scale, kind):
        q, k, v = oa._f64(q), oa._f64(k), oa._f64(v)
        B, lq, Hq, d = q.shape
        lk, Hkv = k.shape[1], k.shape[2]
        o = np.zeros((B, lq, Hq, d))
        lse = np.full((B, Hq, lq), -np.inf)
        r, c = np.arange(lq)[:, None], np.arange(lk)[None, :]
        allowed = np.ones((lq, lk), bool)
        if kind == "masked":
            allowed = c <= r
        elif kind == "strict":
            allowed = (c <= r) if mistake == "strict_keeps_diagonal" else (c < r)
        for b in range(B):
            for h in range(Hq):
                s = scale * (q[b, :, h] @ k[b, :, h // (Hq // Hkv)].T)
                s = np.where(allowed, s, -np.inf)
                for i in range(lq):
                    if not allowed[i].any():
                        if mistake == "empty_row_uniform":
                            o[b, i, h] = v[b, :, h // (Hq // Hkv)].mean(axis=0)
                        continue
                    m = s[i].max()
                    e = np.exp(s[i] - m)
                    o[b, i, h] = e @ v[b, :, h // (Hq // Hkv)] / e.sum()
                    lse[b, h, i] = m + np.log(e.sum()) + (1.0 if mistake == "lse_plus_one" else 0.0)
        return o, lse
    return block


@pytest.mark.parametrize("mistake", ["strict_keeps_diagonal", "empty_row_uniform", "lse_plus_one"])
def test_planted_block_mistake_is_caught(mistake):
    assert any(_fails(pin, _mutant_block(mistake)) for pin in BLOCK_PINS), mistake
    for pin in BLOCK_PINS:
        pin(_mutant_block(None))
