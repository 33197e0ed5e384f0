"""Plain fp64 restatement of the attention backward pass (CPU, slow).

TEST INFRASTRUCTURE ONLY: imported by tests, the smoke check and the CPU
baseline of the benchmark, never by the product path.

The FlashAttention article (section 二, 核心原理 and 重计算) keeps only the
output O and the softmax statistics (max and logsumexp) from the forward pass
and recomputes what the gradients need in the backward pass instead of
storing the L x L attention matrix.  Whatever the method stores, the
gradients it must produce are those of the definition (lnwmold §2.1:
S = scale * Q K^T, A = softmax(S), Output = A V) for a given upstream
gradient dO:

    dV = A^T dO
    dA = dO V^T
    dS = A * (dA - rowsum(A * dA))        (softmax Jacobian, row by row)
    dQ = scale * dS K,   dK = scale * dS^T Q

With grouped-query attention (lnwmold §2.2, contiguous groups) a K/V head's
gradient is the sum over the query heads of its group.  Masked entries of A
are exactly zero and contribute nothing.  ``attention_bwd`` and the row
functions are written from that definition and use no identity the kernels
use.  ``block_attention_bwd`` (one ring visit's share) cannot see the other
blocks' weights, so it writes the Jacobian's row term through the forward
output, rowsum(A * dA) = rowsum(dO * O); it is pinned by summing its shares
over all visits back to ``attention_bwd``.
"""

from __future__ import annotations

import numpy as np

from .attn_fp64 import NEG_INF, _f64, _shapes


def _row_grads(s: np.ndarray, vv: np.ndarray, do: np.ndarray):
    """For score rows s [n, m] (masked entries -inf), values vv [m, d] and
    upstream rows do [n, d]: (A, dS) of the definition."""
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    a = e / e.sum(axis=1, keepdims=True)
    da = do @ vv.T
    ds = a * (da - (a * da).sum(axis=1, keepdims=True))
    return a, ds


def attention_bwd(q, k, v, dout, causal: bool, scale: float):
    """Gradients (dQ, dK, dV) of sum(Output * dout) with respect to q, k, v.
    q, dout [B, L, Hq, d]; k, v [B, L, Hkv, d].  Returns float64 arrays of
    the shapes of q, k, v."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, L, Hq, Hkv, d, g = _shapes(q, k, v)
    if do.shape != q.shape:
        raise ValueError("dout must have the shape of q")
    dq = np.zeros((B, L, Hq, d))
    dk = np.zeros((B, L, Hkv, d))
    dv = np.zeros((B, L, Hkv, d))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            s = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)
            if causal:
                s[np.triu_indices(L, 1)] = NEG_INF
            a, ds = _row_grads(s, v[b, :, kh, :], do[b, :, h, :])
            dv[b, :, kh, :] += a.T @ do[b, :, h, :]
            dq[b, :, h, :] = scale * (ds @ k[b, :, kh, :])
            dk[b, :, kh, :] += scale * (ds.T @ q[b, :, h, :])
    return dq, dk, dv


def attention_bwd_dq_rows(q, k, v, dout, causal: bool, scale: float, bhr, row_block: int = 128):
    """dQ of the definition for the query rows listed in ``bhr`` ([n, 3] of
    (b, h, r)); each row needs only its own scores.  Returns [n, d]."""
    bhr = np.asarray(bhr, dtype=np.int64).reshape(-1, 3)
    B, L, Hq, d = q.shape
    g = Hq // k.shape[2]
    out = np.empty((bhr.shape[0], d))
    keys = bhr[:, 0] * Hq + bhr[:, 1]
    for key in np.unique(keys):
        b, h = int(key // Hq), int(key % Hq)
        kh = h // g
        idx = np.nonzero(keys == key)[0]
        kk = _f64(k[b, :, kh, :])
        vv = _f64(v[b, :, kh, :])
        for s0 in range(0, len(idx), row_block):
            sel = idx[s0:s0 + row_block]
            rs = bhr[sel, 2]
            qq = _f64(q[b, rs.tolist() if hasattr(q, "detach") else rs, h, :])
            dd = _f64(dout[b, rs.tolist() if hasattr(dout, "detach") else rs, h, :])
            s = scale * (qq @ kk.T)
            if causal:
                s[np.arange(L)[None, :] > rs[:, None]] = NEG_INF
            _, ds = _row_grads(s, vv, dd)
            out[sel] = scale * (ds @ kk)
    return out


def attention_bwd_kv_rows(q, k, v, dout, causal: bool, scale: float, bhc, row_block: int = 512):
    """dK and dV of the definition for the key rows listed in ``bhc``
    ([n, 3] of (b, kv_head, c)).  Key row c's gradient sums over every query
    row of every head of its group, so all score rows of those heads are
    formed (in blocks of ``row_block`` query rows).  Returns ([n, d], [n, d])."""
    bhc = np.asarray(bhc, dtype=np.int64).reshape(-1, 3)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    g = Hq // Hkv
    dk = np.zeros((bhc.shape[0], d))
    dv = np.zeros((bhc.shape[0], d))
    keys = bhc[:, 0] * Hkv + bhc[:, 1]
    for key in np.unique(keys):
        b, kh = int(key // Hkv), int(key % Hkv)
        idx = np.nonzero(keys == key)[0]
        cs = bhc[idx, 2]
        kk = _f64(k[b, :, kh, :])
        vv = _f64(v[b, :, kh, :])
        for h in range(kh * g, (kh + 1) * g):
            qh = _f64(q[b, :, h, :])
            dh = _f64(dout[b, :, h, :])
            for r0 in range(0, L, row_block):
                r1 = min(L, r0 + row_block)
                s = scale * (qh[r0:r1] @ kk.T)
                if causal:
                    s[np.arange(L)[None, :] > np.arange(r0, r1)[:, None]] = NEG_INF
                a, ds = _row_grads(s, vv, dh[r0:r1])
                dv[idx] += a[:, cs].T @ dh[r0:r1]
                dk[idx] += scale * (ds[:, cs].T @ qh[r0:r1])
    return dk, dv


def block_attention_bwd(q, k, v, out, dout, lse, scale: float, kind: str):
    """One ring visit's share of the gradients: the query block (rows r, with
    their forward output ``out`` and natural-log ``lse`` over the WHOLE
    sequence) against one K/V block under the visit mask ``kind`` of
    ``attn_fp64.block_attention`` ("full", "masked" keys c <= r, "strict"
    keys c < r).  With A the rows' attention weights restricted to this
    block's keys (A = exp(scale q.k - lse), the block's columns of the full
    softmax) and the Jacobian's row term rowsum(A_full * dA_full) written as
    rowsum(dO * O) (O = A_full V):

        dV_part = A^T dO,   dS = A * (dO V^T - rowsum(dO * O))
        dQ_part = scale dS K,   dK_part = scale dS^T Q

    Summed over every K/V block a query block visits, the parts are the
    gradients of :func:`attention_bwd` (the pin of this function).
    q, out, dout [B, lq, Hq, d]; k, v [B, lk, Hkv, d]; lse [B, Hq, lq].
    Returns float64 (dq_part, dk_part, dv_part)."""
    q, k, v, o, do, lse = (_f64(x) for x in (q, k, v, out, dout, lse))
    B, lq, Hq, d = q.shape
    lk, Hkv = k.shape[1], k.shape[2]
    if kind not in ("full", "masked", "strict"):
        raise ValueError(f"unknown visit kind {kind!r}")
    if kind != "full" and lq != lk:
        raise ValueError("masked visits need equal block lengths")
    g = Hq // Hkv
    rows = np.arange(lq)[:, None]
    cols = np.arange(lk)[None, :]
    allowed = np.ones((lq, lk), dtype=bool)
    if kind == "masked":
        allowed = cols <= rows
    elif kind == "strict":
        allowed = cols < rows
    dq = np.zeros((B, lq, Hq, d))
    dk = np.zeros((B, lk, Hkv, d))
    dv = np.zeros((B, lk, Hkv, d))
    for b in range(B):
        for h in range(Hq):
            kh = h // g
            s = scale * (q[b, :, h, :] @ k[b, :, kh, :].T)
            a = np.where(allowed, np.exp(s - lse[b, h][:, None]), 0.0)
            rterm = (do[b, :, h, :] * o[b, :, h, :]).sum(axis=1, keepdims=True)
            ds = a * (do[b, :, h, :] @ v[b, :, kh, :].T - rterm)
            dv[b, :, kh, :] += a.T @ do[b, :, h, :]
            dq[b, :, h, :] = scale * (ds @ k[b, :, kh, :])
            dk[b, :, kh, :] += scale * (ds.T @ q[b, :, h, :])
    return dq, dk, dv
