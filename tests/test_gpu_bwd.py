"""GPU parity of the backward pass (ring_attn_bwd, through the C ABI) against
the fp64 oracle's gradients of the same definition."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from parity import compare_grad

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


def fwd_bwd(api, q, k, v, do, n_ring, causal, scale=None):
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = api.fwd(qd, kd, vd, n_ring, causal, scale)
    dq, dk, dv = api.bwd(qd, kd, vd, out, dod, lse, n_ring, causal, scale)
    api.check_status()
    return dq.cpu(), dk.cpu(), dv.cpu()


def full_check(api, B, Hq, Hkv, L, d, n_ring, causal, seed, what):
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, L, d, seed=seed)
    do = make_grad_output(B, L, Hq, d, seed=seed)
    scale = 1.0 / d ** 0.5
    got = fwd_bwd(api, q, k, v, do, n_ring, causal, scale)
    ref = oracle.attention_bwd(q, k, v, do, causal, scale)
    return [compare_grad(g, r, f"{what} {name}") for g, r, name in zip(got, ref, "qkv")]


# (B, Hq, Hkv, L, d, n_ring, causal): several tiles, ragged blocks, GQA with
# even and odd groups, ring sizes 1..5, a single-row sequence
SMALL = [
    (1, 1, 1, 128, 128, 1, True),
    (1, 2, 2, 256, 128, 2, True),
    (1, 2, 2, 256, 128, 2, False),
    (2, 4, 2, 384, 64, 3, True),
    (1, 4, 1, 600, 128, 3, True),      # blocks of 200 rows: a full tile + 72
    (1, 2, 2, 200, 64, 5, False),      # blocks of 40 rows
    (1, 3, 1, 512, 128, 4, True),      # group of 3
    (1, 2, 2, 1024, 128, 4, True),
    (1, 1, 1, 1, 64, 1, True),         # one row
]


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n_ring,causal", SMALL)
def test_bwd_small_shapes(ra, B, Hq, Hkv, L, d, n_ring, causal):
    full_check(ra, B, Hq, Hkv, L, d, n_ring, causal, seed=7 * L + d + n_ring,
               what=f"{(B, Hq, Hkv, L, d, n_ring, causal)}")


def test_bwd_workload_l512_d64_noncausal(ra):
    full_check(ra, 1, 1, 1, 512, 64, 4, False, seed=0, what="l512")


def test_bwd_workload_l8k_h8_causal(ra):
    """The 8K-token causal workload (B 2, 8 heads, d 128, 4 ring blocks):
    every gradient element against the oracle."""
    from ring_attention_ordered_b200.inputs import WORKLOADS
    w = WORKLOADS["l8k_h8_causal"]
    full_check(ra, w.B, w.Hq, w.Hkv, w.L, w.d, w.n_ring, w.causal, seed=w.seed, what=w.name)


def test_bwd_gqa_workload_dq_rows_and_one_kv_head(ra):
    """The 32K-token GQA workload (32 query heads on 8 K/V heads, keys x2):
    sampled dQ rows plus rows around every ring-block boundary, and dK/dV
    rows of K/V head 0 around the block boundaries (each needs every score
    row of the group's four heads)."""
    from ring_attention_ordered_b200.inputs import WORKLOADS, make_grad_output, sample_rows, workload_inputs
    w = WORKLOADS["l32k_gqa4_causal"]
    q, k, v = workload_inputs(w)
    do = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = ra.fwd(qd, kd, vd, w.n_ring, w.causal, w.scale)
    dq, dk, dv = ra.bwd(qd, kd, vd, out, dod, lse, w.n_ring, w.causal, w.scale)
    ra.check_status()
    del qd, kd, vd, dod, out, lse
    lb = w.block_len
    edges = sorted({r for i in range(w.n_ring + 1) for r in (i * lb - 1, i * lb, i * lb + 127)
                    if 0 <= r < w.L})
    bhr = np.concatenate([sample_rows(w, 512),
                          np.array([[0, h, r] for h in (0, w.Hq - 1) for r in edges], np.int64)])
    ref = oracle.attention_bwd_dq_rows(q, k, v, do, w.causal, w.scale, bhr)
    b, h, r = (torch.from_numpy(bhr[:, i]).cuda() for i in range(3))
    compare_grad(dq[b, r, h, :], ref, "l32k dQ rows")
    bhc = np.array([[0, 0, r] for r in edges], np.int64)
    rk, rv = oracle.attention_bwd_kv_rows(q, k, v, do, w.causal, w.scale, bhc)
    c = torch.from_numpy(bhc[:, 2]).cuda()
    compare_grad(dk[0, c, 0, :], rk, "l32k dK rows")
    compare_grad(dv[0, c, 0, :], rv, "l32k dV rows")


def test_bwd_deterministic_and_grid_invariant(ra):
    """Every gradient element is accumulated by one CTA in a fixed order, so
    the result is bitwise the same whatever the number of CTAs."""
    from ring_attention_ordered_b200 import _lib
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    q, k, v = make_inputs(2, 4, 2, 1024, 128, seed=21)
    do = make_grad_output(2, 1024, 4, 128, seed=21)
    ref = fwd_bwd(ra, q, k, v, do, 4, True)
    try:
        for cap in (1, 5, 0):
            _lib.ring_attn_set_max_ctas(cap)
            got = fwd_bwd(ra, q, k, v, do, 4, True)
            for a, b in zip(got, ref):
                assert torch.equal(a, b), cap
    finally:
        _lib.ring_attn_set_max_ctas(0)


def test_bwd_bounded_wait_reports_timeout_and_recovers(ra):
    from ring_attention_ordered_b200 import _lib
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    q, k, v = (t.cuda() for t in make_inputs(1, 2, 2, 512, 128, seed=22))
    do = make_grad_output(1, 512, 2, 128, seed=22).cuda()
    out, lse = ra.fwd(q, k, v, 4, True)
    ra.check_status()
    try:
        _lib.ring_attn_set_wait_limit_ns(200_000_000)
        _lib.ring_attn_debug_inject(1)
        ra.bwd(q, k, v, out, do, lse, 4, True)
        with pytest.raises(_lib.RingAttnError) as ei:
            ra.check_status()
        assert ei.value.status == _lib.RA_ERR_TIMEOUT
    finally:
        _lib.ring_attn_debug_inject(0)
        _lib.ring_attn_set_wait_limit_ns(0)
    full_check(ra, 1, 2, 2, 512, 128, 4, True, seed=22, what="after timeout")


def test_bwd_short_workspace_is_rejected(ra):
    from ring_attention_ordered_b200 import _lib
    q = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 256), dtype=torch.float32, device="cuda")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.RingAttnError) as ei:
        ra.bwd(q, q.clone(), q.clone(), q.clone(), q.clone(), lse, 2, True, workspace=ws)
    assert ei.value.status == _lib.RA_ERR_INVALID_ARG


@pytest.mark.parametrize("name,n_sample", [("l128k_h32_causal", 256), ("l1m_gqa4_sink_causal", 256)])
def test_bwd_large_workloads_dq_rows(ra, name, n_sample):
    """The 128K and the 1M-token (attention-sink, GQA) workloads at full
    size: sampled dQ rows and rows at every ring-block boundary of the first
    and last head against the oracle (each dQ row needs only its own scores);
    dK and dV, which need every query row of a group, are checked on the
    smaller workloads."""
    from ring_attention_ordered_b200.inputs import WORKLOADS, make_grad_output, sample_rows, workload_inputs
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w)
    do = make_grad_output(w.B, w.L, w.Hq, w.d, w.seed)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    out, lse = ra.fwd(qd, kd, vd, w.n_ring, w.causal, w.scale)
    dq, dk, dv = ra.bwd(qd, kd, vd, out, dod, lse, w.n_ring, w.causal, w.scale)
    ra.check_status()
    assert torch.isfinite(dk).all() and torch.isfinite(dv).all()
    del qd, kd, vd, dod, out, lse, dk, dv
    lb = w.block_len
    edges = sorted({r for i in range(w.n_ring + 1) for r in (i * lb - 1, i * lb) if 0 <= r < w.L})
    bhr = np.concatenate([sample_rows(w, n_sample, seed=w.seed + 1),
                          np.array([[0, h, r] for h in (0, w.Hq - 1) for r in edges], np.int64)])
    ref = oracle.attention_bwd_dq_rows(q, k, v, do, w.causal, w.scale, bhr)
    b, h, r = (torch.from_numpy(bhr[:, i]).cuda() for i in range(3))
    compare_grad(dq[b, r, h, :], ref, f"{name} dQ rows")


def test_autograd_function_matches_oracle(ra):
    """api.attention under torch.autograd: output and q, k, v gradients of a
    GQA causal problem against the oracle."""
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    q, k, v = make_inputs(1, 4, 2, 768, 128, seed=61)
    do = make_grad_output(1, 768, 4, 128, seed=61)
    qd, kd, vd = (t.cuda().requires_grad_() for t in (q, k, v))
    out = ra.attention(qd, kd, vd, 3, True)
    out.backward(do.cuda())
    ra.check_status()
    scale = 1.0 / 128 ** 0.5
    o_ref, _ = oracle.attention(q, k, v, True, scale)
    err = np.abs(out.detach().float().cpu().numpy() - o_ref)
    assert err.max() <= 1.6e-2 and err.mean() <= 1e-3
    ref = oracle.attention_bwd(q, k, v, do, True, scale)
    for g_, r_, n in zip((qd.grad, kd.grad, vd.grad), ref, "qkv"):
        compare_grad(g_, r_, f"autograd d{n}")


def test_side_stream_calls_match_the_current_stream(ra):
    """fwd and bwd launched on a side stream, with their outputs and the
    backward's workspace allocated by the wrapper, give bitwise the results of
    the same calls on the current stream.  Right after the calls return, the
    current stream allocates and fills buffers of the workspace's size: had
    the workspace been allocated on the current stream, the caching allocator
    could hand its block to them while the side stream's kernels still use it."""
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    B, Hq, Hkv, L, d, n_ring = 1, 8, 2, 4096, 128, 4
    q, k, v = (t.cuda() for t in make_inputs(B, Hq, Hkv, L, d, seed=51))
    do = make_grad_output(B, L, Hq, d, 51).cuda()
    out0, lse0 = ra.fwd(q, k, v, n_ring, True)
    ref = ra.bwd(q, k, v, out0, do, lse0, n_ring, True)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    out1, lse1 = ra.fwd(q, k, v, n_ring, True, stream=side)
    got = ra.bwd(q, k, v, out1, do, lse1, n_ring, True, stream=side)
    ws_bytes = B * Hq * L * 4
    junk = [torch.full((ws_bytes // 4,), float("nan"), device="cuda") for _ in range(8)]
    side.synchronize()
    torch.cuda.synchronize()
    ra.check_status(side)
    assert torch.equal(out1, out0) and torch.equal(lse1, lse0)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    del junk


def test_bwd_work_queue_concurrent_streams_and_graph_replay(ra):
    """Both backward kernels take units from a per-launch queue counter (one
    of a ring of device counters, zeroed by a stream-ordered memset).  Calls
    on two streams at once, and a backward captured in a CUDA graph and
    replayed, must give bitwise the results of plain calls."""
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    shapes = [(1, 8, 2, 2048, 128, 63), (2, 4, 4, 1024, 128, 64)]
    dev = []
    for B, Hq, Hkv, L, d, seed in shapes:
        q, k, v = (t.cuda() for t in make_inputs(B, Hq, Hkv, L, d, seed=seed))
        do = make_grad_output(B, L, Hq, d, seed).cuda()
        out, lse = ra.fwd(q, k, v, 4, True)
        dev.append((q, k, v, out, do, lse))
    ref = [ra.bwd(q, k, v, out, do, lse, 4, True) for q, k, v, out, do, lse in dev]
    torch.cuda.synchronize()
    # concurrent: both problems in flight on their own streams, three times
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    got = []
    for _ in range(3):
        for (q, k, v, out, do, lse), s in zip(dev, streams):
            got.append(ra.bwd(q, k, v, out, do, lse, 4, True, stream=s))
    for s in streams:
        s.synchronize()
    ra.check_status()
    for i, g in enumerate(got):
        for a, b in zip(g, ref[i % 2]):
            assert torch.equal(a, b)
    # graph: both counter resets are captured with their launches
    q, k, v, out, do, lse = dev[0]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, ra._lib.ring_attn_bwd_workspace_size(q.shape[0], q.shape[2], q.shape[1])),
                     dtype=torch.uint8, device="cuda")
    ra.bwd(q, k, v, out, do, lse, 4, True, dq=dq, dk=dk, dv=dv, workspace=ws)   # outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ra.bwd(q, k, v, out, do, lse, 4, True, dq=dq, dk=dk, dv=dv, workspace=ws,
               stream=torch.cuda.current_stream())
    for _ in range(3):
        for t in (dq, dk, dv):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        ra.check_status()
        for a, b in zip((dq, dk, dv), ref[0]):
            assert torch.equal(a, b)
    del g
