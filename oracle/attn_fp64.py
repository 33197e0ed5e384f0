"""Plain fp64 restatement of ring-ordered blockwise attention (CPU, slow).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the CPU
baseline of the benchmark, never by the product path.

Readings of the pages taken here (each one is the plainest reading that the
rest of the pages support):

* Tensors: ``q`` is [B, L, Hq, d]; ``k`` and ``v`` are [B, L, Hkv, d].  Any
  real dtype is accepted and converted exactly to float64, so bf16 inputs are
  compared on their rounded values.
* Scores are ``scale * q . k``; the pages use scale = 1/sqrt(d)
  ("Ring Attention 环注意力", L4 §4.3 ``ring_attention_step``; lnwmold page
  §2.1 S = QK^T/sqrt(d)).  Callers pass the scale explicitly.
* Causal masking keeps keys c <= r (query row r, equal lengths); at block
  level host i attends K_{<=i} ("Ring Attention 环注意力", L4 §4.5,
  limitation 2).
* GQA groups query heads contiguously: head h reads KV head h // (Hq/Hkv)
  (lnwmold page §2.2, MQA/GQA: several heads form a group that shares K/V).
* The log-sum-exp statistic is in natural log (FlashAttention article,
  FlashAttention-2 改进: only the logsumexp statistic is stored).

Functions are written row by row from the definition; the only batching is
over independent query rows (a library matmul computes the scores of several
rows at once), which changes no per-row arithmetic.
"""

from __future__ import annotations

import math

import numpy as np

NEG_INF = float("-inf")


def _f64(x) -> np.ndarray:
    # torch tensors (bf16 included) are widened through float32, which holds
    # every bf16 value exactly
    if hasattr(x, "detach") and hasattr(x, "float"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def _shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, L, H, d]")
    B, L, Hq, d = q.shape
    Bk, Lk, Hkv, dk = k.shape
    if (Bk, Lk, dk) != (B, L, d) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{q.shape} k{k.shape} v{v.shape}")
    if Hkv < 1 or Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return B, L, Hq, Hkv, d, Hq // Hkv


def _softmax_weighted_sum(s: np.ndarray, vals: np.ndarray):
    """For each row of scores ``s`` (masked entries are -inf) return
    (sum_c exp(s_c - M) v_c / Z, M + ln Z) with M = max_c s_c and
    Z = sum_c exp(s_c - M): the standard softmax-weighted sum (lnwmold page
    §2.1: A = softmax(S), Output = AV) and the log-sum-exp of the row."""
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    z = e.sum(axis=1)
    o = (e @ vals) / z[:, None]
    return o, m + np.log(z)


def attention(q, k, v, causal: bool, scale: float, row_block: int = 1024):
    """Full attention softmax(scale * Q K^T + mask) V and the per-row LSE.

    The definition the ring method must reproduce exactly: the FlashAttention
    article (section 二) states that the blockwise method is exact, equal in
    value to standard attention, and lnwmold §2.1 defines that attention.
    Returns ``O`` [B, L, Hq, d] and ``lse`` [B, Hq, L], both float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, Hq, Hkv, d, g = _shapes(q, k, v)
    out = np.empty((B, L, Hq, d))
    lse = np.empty((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for r0 in range(0, L, row_block):
                r1 = min(L, r0 + row_block)
                # keys past r1-1 are masked for every row of this batch under
                # causal masking; they would contribute exp(-inf) = 0
                nk = r1 if causal else L
                kk = k[b, :nk, kh, :]
                s = scale * (q[b, r0:r1, h, :] @ kk.T)
                if causal:
                    rows = np.arange(r0, r1)[:, None]
                    cols = np.arange(nk)[None, :]
                    s[cols > rows] = NEG_INF
                o, l_ = _softmax_weighted_sum(s, v[b, :nk, kh, :])
                out[b, r0:r1, h, :] = o
                lse[b, h, r0:r1] = l_
    return out, lse


def attention_rows(q, k, v, causal: bool, scale: float, bhr, row_block: int = 128):
    """The same definition as :func:`attention`, evaluated only for the
    query rows listed in ``bhr`` (an int array [n, 3] of (b, h, r)).

    Returns ``O`` [n, d] and ``lse`` [n] in the order of ``bhr``.  Used for
    the large workloads, where the full output is out of reach on a CPU.
    Inputs may be any array type with numpy-style indexing (converted per head
    to float64, so a large bf16 tensor is never widened whole).
    """
    bhr = np.asarray(bhr, dtype=np.int64).reshape(-1, 3)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    n = bhr.shape[0]
    out = np.empty((n, d))
    lse = np.empty(n)
    keys = bhr[:, 0] * Hq + bhr[:, 1]
    for key in np.unique(keys):
        b, h = int(key // Hq), int(key % Hq)
        kh = h // g
        idx = np.nonzero(keys == key)[0]
        idx = idx[np.argsort(bhr[idx, 2], kind="stable")]
        kk_all = _f64(k[b, :, kh, :])
        vv_all = _f64(v[b, :, kh, :])
        for s0 in range(0, len(idx), row_block):
            sel = idx[s0:s0 + row_block]
            rs = bhr[sel, 2]
            nk = int(rs.max()) + 1 if causal else L
            qq = _f64(q[b, rs.tolist() if hasattr(q, "detach") else rs, h, :])
            s = scale * (qq @ kk_all[:nk].T)
            if causal:
                s[np.arange(nk)[None, :] > rs[:, None]] = NEG_INF
            o, l_ = _softmax_weighted_sum(s, vv_all[:nk])
            out[sel] = o
            lse[sel] = l_
    return out, lse


def attention_probs(q, k, causal: bool, scale: float):
    """Attention weights A = softmax(scale * Q K^T + mask) as [B, Hq, L, L]
    (lnwmold §2.1).  Tiny inputs only; exposes the row-sum invariant."""
    q, k = _f64(q), _f64(k)
    B, L, Hq, d = q.shape
    g = Hq // k.shape[2]
    p = np.empty((B, Hq, L, L))
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, :, h, :] @ k[b, :, h // g, :].T)
            if causal:
                s[np.triu_indices(L, 1)] = NEG_INF
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            p[b, h] = e / e.sum(axis=1, keepdims=True)
    return p


def brute_attention(q, k, v, causal: bool, scale: float):
    """Pure-Python triple loop with exactly rounded sums (math.fsum): the
    definition of lnwmold §2.1 with nothing vectorised.  Tiny inputs only."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, Hq, Hkv, d, g = _shapes(q, k, v)
    out = np.zeros((B, L, Hq, d))
    lse = np.zeros((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for r in range(L):
                cols = range(r + 1) if causal else range(L)
                s = [scale * math.fsum(q[b, r, h, t] * k[b, c, kh, t] for t in range(d))
                     for c in cols]
                mx = max(s)
                e = [math.exp(x - mx) for x in s]
                z = math.fsum(e)
                for t in range(d):
                    out[b, r, h, t] = math.fsum(e[i] * v[b, c, kh, t]
                                                for i, c in enumerate(cols)) / z
                lse[b, h, r] = mx + math.log(z)
    return out, lse


def ring_order(i: int, n_ring: int):
    """Blocks host ``i`` holds at steps t = 0..N-1: K/V block (i - t) mod N.

    "Ring Attention 环注意力", L3 definition (at step t GPU i receives
    K_{(i-t)%N}, V_{(i-t)%N} from GPU i-1) and the N=4 picture of L4 §4.2."""
    if n_ring < 1 or not 0 <= i < n_ring:
        raise ValueError("need 0 <= i < n_ring")
    return [(i - t) % n_ring for t in range(n_ring)]


def ring_visits(i: int, n_ring: int, causal: bool):
    """The visits host ``i`` computes, in ring order, as (t, j, kind).

    Under causal masking Q_i attends only K_{<=i} ("Ring Attention 环注意力",
    L4 §4.5, limitation 2), so blocks j > i are skipped, block j == i is
    masked on its diagonal ("masked") and blocks j < i run in full ("full").
    Without masking every block is "full"."""
    visits = []
    for t, j in enumerate(ring_order(i, n_ring)):
        if causal and j > i:
            continue
        visits.append((t, j, "masked" if (causal and j == i) else "full"))
    return visits


def _block_scores(qi, kj, scale, kind):
    s = scale * (qi @ kj.T)
    if kind == "masked":
        s[np.triu_indices(s.shape[0], 1)] = NEG_INF
    return s


def block_attention(q, k, v, scale: float, kind: str):
    """Exact attention of one query block against one K/V block, as a partial
    result (o, lse) over the keys the visit allows -- what one host computes on
    one ring step before folding it into its output ("Ring Attention 环注意力",
    L4 §4.2 steps 1-2).  Local rows r of the query block, c of the K/V block:

    * ``"full"``: every key (an earlier block, or no causal mask);
    * ``"masked"``: keys c <= r (the host's own block under causal masking);
    * ``"strict"``: keys c < r (a striped layout's block from a later host,
      "Striped Attention" in L4 §4.8: its key at local row r comes after the
      query in the sequence).

    A row with no allowed key is the empty partial: o = 0, lse = -inf.
    q [B, lq, Hq, d], k/v [B, lk, Hkv, d] (lq == lk unless ``"full"``).
    Returns o [B, lq, Hq, d], lse [B, Hq, lq] in float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, lq, Hq, d = q.shape
    _, lk, Hkv, _ = k.shape
    if kind not in ("full", "masked", "strict"):
        raise ValueError(f"unknown visit kind {kind!r}")
    if kind != "full" and lq != lk:
        raise ValueError("masked visits need equal block lengths")
    g = Hq // Hkv
    o = np.zeros((B, lq, Hq, d))
    lse = np.full((B, Hq, lq), NEG_INF)
    rows = np.arange(lq)[:, None]
    cols = np.arange(lk)[None, :]
    allowed = np.ones((lq, lk), dtype=bool)
    if kind == "masked":
        allowed = cols <= rows
    elif kind == "strict":
        allowed = cols < rows
    live = allowed.any(axis=1)
    for b in range(B):
        for h in range(Hq):
            s = scale * (q[b, :, h, :] @ k[b, :, h // g, :].T)
            s = np.where(allowed, s, NEG_INF)[live]
            if s.shape[0] == 0:
                continue
            o_r, l_r = _softmax_weighted_sum(s, v[b, :, h // g, :])
            o[b, live, h, :] = o_r
            lse[b, h, live] = l_r
    return o, lse


def ring_attention(q, k, v, n_ring: int, causal: bool, scale: float):
    """Ring attention emulated on one host, with the running accumulator.

    The sequence is cut into N equal blocks of l = L/N rows ("Ring Attention
    环注意力", L4 §4.2 setup).  Host i keeps Q_i and, over the ring visits of
    :func:`ring_visits`, a running row max m, row sum l and unnormalised
    output O.  Each visit follows L4 §4.3 ``ring_attention_step`` read row by
    row, which is the FlashAttention recurrence (FlashAttention article, 核心
    原理: accumulated max and exponential sum):

        S = scale * Q_i K_j^T            (diagonal-masked on the "masked" visit)
        m' = max(m, rowmax S)
        P = exp(S - m')
        l' = exp(m - m') * l + rowsum P
        O' = exp(m - m') * O + P V_j

    and after the last visit O / l and lse = m + ln l.  (The listing on the
    page takes a scalar max, omits the subtraction of m' inside exp and
    divides by l at every step; only the row-wise reading with one final
    division reproduces exact attention, which the pages say the method is.)
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, Hq, Hkv, d, g = _shapes(q, k, v)
    if n_ring < 1 or L % n_ring != 0:
        raise ValueError("L must split into n_ring equal blocks")
    lb = L // n_ring
    out = np.empty((B, L, Hq, d))
    lse = np.empty((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i in range(n_ring):
                qi = q[b, i * lb:(i + 1) * lb, h, :]
                m = np.full(lb, NEG_INF)
                lsum = np.zeros(lb)
                o = np.zeros((lb, d))
                for _, j, kind in ring_visits(i, n_ring, causal):
                    kj = k[b, j * lb:(j + 1) * lb, kh, :]
                    vj = v[b, j * lb:(j + 1) * lb, kh, :]
                    s = _block_scores(qi, kj, scale, kind)
                    m_new = np.maximum(m, s.max(axis=1))
                    alpha = np.exp(m - m_new)
                    p = np.exp(s - m_new[:, None])
                    lsum = alpha * lsum + p.sum(axis=1)
                    o = alpha[:, None] * o + p @ vj
                    m = m_new
                out[b, i * lb:(i + 1) * lb, h, :] = o / lsum[:, None]
                lse[b, h, i * lb:(i + 1) * lb] = m + np.log(lsum)
    return out, lse


def merge(o_a, lse_a, o_b, lse_b):
    """Fold two partial results over disjoint key sets into one.

    The pages describe the fold as accumulating each step's FlashAttention
    result into O_i ("Ring Attention 环注意力", L4 §4.2, step 2) and keep only
    the logsumexp statistic (FlashAttention article, FlashAttention-2 改进); the formula
    they leave implicit is the log-sum-exp combination

        M = max(lse_a, lse_b),  w = exp(lse - M)
        lse = M + ln(w_a + w_b),  o = (w_a o_a + w_b o_b) / (w_a + w_b).

    An empty partial (lse = -inf) contributes nothing: the other side is
    returned exactly, and two empty partials give o = 0, lse = -inf.  NaN
    propagates.  Shapes: o [..., d], lse [...].
    """
    oa, ob = _f64(o_a), _f64(o_b)
    la, lb = _f64(lse_a), _f64(lse_b)
    mx = np.maximum(la, lb)
    empty = mx == NEG_INF
    m0 = np.where(empty, 0.0, mx)
    wa = np.exp(la - m0)
    wb = np.exp(lb - m0)
    den = wa + wb
    with np.errstate(invalid="ignore", divide="ignore"):
        ta = np.where((wa == 0)[..., None], 0.0, wa[..., None] * oa)
        tb = np.where((wb == 0)[..., None], 0.0, wb[..., None] * ob)
        o = (ta + tb) / den[..., None]
        lse = m0 + np.log(den)
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, NEG_INF, lse)
    return o, lse


def ring_attention_merged(q, k, v, n_ring: int, causal: bool, scale: float):
    """Ring attention in the "partial result per visit" form: every visit
    yields its own exact (O_t, lse_t) over block j, and host i folds them in
    ring order with :func:`merge`, starting from the empty partial
    ("Ring Attention 环注意力", L4 §4.2, step 2: each step's blockwise result
    is accumulated into O_i)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, L, Hq, Hkv, d, g = _shapes(q, k, v)
    if n_ring < 1 or L % n_ring != 0:
        raise ValueError("L must split into n_ring equal blocks")
    lb = L // n_ring
    out = np.empty((B, L, Hq, d))
    lse = np.empty((B, Hq, L))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            for i in range(n_ring):
                qi = q[b, i * lb:(i + 1) * lb, h, :]
                o = np.zeros((lb, d))
                l_ = np.full(lb, NEG_INF)
                for _, j, kind in ring_visits(i, n_ring, causal):
                    s = _block_scores(qi, k[b, j * lb:(j + 1) * lb, kh, :], scale, kind)
                    o_t, l_t = _softmax_weighted_sum(s, v[b, j * lb:(j + 1) * lb, kh, :])
                    o, l_ = merge(o, l_, o_t, l_t)
                out[b, i * lb:(i + 1) * lb, h, :] = o
                lse[b, h, i * lb:(i + 1) * lb] = l_
    return out, lse


def causal_pair_counts(n_ring: int):
    """(computed, masked, skipped) block pairs over all hosts under causal
    masking, counted from :func:`ring_visits` ("Ring Attention 环注意力",
    L4 §4.5 limitation 2: the later K blocks are of no use to earlier Q)."""
    computed = masked = 0
    for i in range(n_ring):
        for _, _, kind in ring_visits(i, n_ring, True):
            computed += 1
            masked += kind == "masked"
    return computed, masked, n_ring * n_ring - computed


def kv_bytes_per_ring_step(block_len: int, heads: int, d: int, elem_bytes: int = 2) -> int:
    """Bytes of one K/V block pair handed to the next host per ring step:
    K and V, each block_len x heads x d elements (interview page on long-text
    optimisation, follow-up 3: 2 x 16K x 128 x 32 x 2 bytes per block)."""
    return 2 * block_len * heads * d * elem_bytes
