"""GPU parity of ring_attn_fwd (through the C ABI) against the fp64 oracle."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity import compare, compare_lse, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


def run(api, q, k, v, n_ring, causal, scale=None):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = api.fwd(qd, kd, vd, n_ring, causal, scale)
    api.check_status()
    return out.cpu(), lse.cpu()


def full_compare(api, q, k, v, n_ring, causal, scale=None, what=""):
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out, lse = run(api, q, k, v, n_ring, causal, scale)
    o_ref, l_ref = oracle.attention(q, k, v, causal, scale)
    return compare(out, lse, o_ref, l_ref, what)


# (B, Hq, Hkv, L, d, n_ring, causal): several tiles, ring sizes 1..16, GQA
# groups 1..4 (odd group included), ragged blocks (not a multiple of 128
# rows, shorter than one tile), tiny and single-row sequences
SMALL = [
    (1, 1, 1, 128, 64, 1, False),
    (1, 1, 1, 128, 128, 1, True),
    (1, 2, 2, 512, 128, 4, True),
    (1, 2, 2, 512, 128, 4, False),
    (2, 4, 1, 768, 128, 3, True),
    (1, 4, 2, 1024, 64, 2, True),
    (1, 3, 1, 512, 128, 2, True),
    (1, 6, 2, 256, 128, 1, False),
    (1, 2, 2, 1536, 128, 6, True),
    (1, 1, 1, 2048, 128, 16, True),
    (1, 1, 1, 2048, 64, 16, False),
    (1, 2, 1, 600, 128, 3, True),      # blocks of 200 rows: a full tile + 72
    (2, 4, 2, 200, 64, 5, False),      # blocks of 40 rows
    (1, 2, 2, 200, 128, 5, True),
    (1, 1, 1, 1, 64, 1, False),        # one row
    (1, 1, 1, 3, 128, 3, True),        # one row per block
    (3, 2, 2, 384, 128, 2, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n_ring,causal", SMALL)
def test_small_shapes(ra, B, Hq, Hkv, L, d, n_ring, causal):
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(B, Hq, Hkv, L, d, seed=B * 1000 + L + d + n_ring)
    full_compare(ra, q, k, v, n_ring, causal, what=f"{(B, Hq, Hkv, L, d, n_ring, causal)}")


def test_workload_l512_d64_noncausal(ra):
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["l512_d64_noncausal"]
    q, k, v = workload_inputs(w)
    full_compare(ra, q, k, v, w.n_ring, w.causal, w.scale, w.name)


def test_workload_l8k_h8_causal_all_rows(ra):
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["l8k_h8_causal"]
    q, k, v = workload_inputs(w)
    full_compare(ra, q, k, v, w.n_ring, w.causal, w.scale, w.name)


def boundary_rows(w, heads):
    """Rows around every ring-block boundary and the sequence ends."""
    rows = set()
    lb = w.block_len
    for i in range(w.n_ring + 1):
        for r in (i * lb - 2, i * lb - 1, i * lb, i * lb + 1, i * lb + 127, i * lb + 128):
            if 0 <= r < w.L:
                rows.add(r)
    return np.array([[b, h, r] for b in range(w.B) for h in heads for r in sorted(rows)],
                    dtype=np.int64)


def _run_workload(ra, name):
    from ring_attention_ordered_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS[name]
    q, k, v = workload_inputs(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out, lse = ra.fwd(qd, kd, vd, w.n_ring, w.causal, w.scale)
    ra.check_status()
    del qd, kd, vd
    return w, (q, k, v), out, lse


def _check_rows(w, qkv, out, lse, bhr, what):
    from oracle_pool import attention_rows_parallel
    o_ref, l_ref = attention_rows_parallel(*qkv, w.causal, w.scale, bhr)
    b, h, r = (torch.from_numpy(bhr[:, i]).cuda() for i in range(3))
    compare(out[b, r, h, :], lse[b, h, r], o_ref, l_ref, what)


def test_workload_l32k_gqa4_causal_all_rows(ra):
    """Every row of every head of the GQA 32K workload (K x2: sharp peaks)."""
    w, qkv, out, lse = _run_workload(ra, "l32k_gqa4_causal")
    rows = np.arange(w.L, dtype=np.int64)
    bhr = np.array([[b, h, 0] for b in range(w.B) for h in range(w.Hq)], dtype=np.int64)
    bhr = np.repeat(bhr, w.L, axis=0)
    bhr[:, 2] = np.tile(rows, w.B * w.Hq)
    _check_rows(w, qkv, out, lse, bhr, f"{w.name} all {len(bhr)} rows")


def test_workload_l128k_h32_causal_rows_and_full_lse(ra, golden_dir):
    """The headline workload: 4096 rows drawn uniformly (every element of O
    and the LSE), rows around every ring-block boundary of the first and last
    head, and the complete LSE of heads 0 and 1 against the stored oracle
    result (written by tests/golden/make_l128k_lse.py)."""
    import hashlib
    import json
    import os
    from ring_attention_ordered_b200.inputs import sample_rows
    w, qkv, out, lse = _run_workload(ra, "l128k_h32_causal")
    # complete LSE of heads 0 and 1
    meta = json.load(open(os.path.join(golden_dir, "l128k_h32_causal_lse_h01.json")))
    ref = np.load(os.path.join(golden_dir, "l128k_h32_causal_lse_h01.npy"))
    assert hashlib.sha256(ref.tobytes()).hexdigest() == meta["array_sha256"]
    q, k, v = qkv
    digest = hashlib.sha256()
    for hd in meta["heads"]:
        for t, i in ((q, hd), (k, hd // w.group), (v, hd // w.group)):
            digest.update(t[:, :, i].contiguous().view(torch.int16).numpy().tobytes())
    assert digest.hexdigest() == meta["inputs_sha256"], "inputs differ from the stored ones"
    compare_lse(lse[0, meta["heads"]], ref, f"{w.name} complete LSE of heads {meta['heads']}")
    bhr = np.concatenate([sample_rows(w, 4096), boundary_rows(w, [0, w.Hq - 1])])
    _check_rows(w, qkv, out, lse, bhr, f"{w.name} 4096 uniform + boundary rows")


def test_workload_l1m_gqa4_sink_causal_rows_per_head(ra):
    """The 1M-token sink workload: 1024 rows drawn per head (8192), plus rows
    around every ring-block boundary of the first and last head."""
    from ring_attention_ordered_b200.inputs import sample_rows_per_head
    w, qkv, out, lse = _run_workload(ra, "l1m_gqa4_sink_causal")
    bhr = np.concatenate([sample_rows_per_head(w, 1024), boundary_rows(w, [0, w.Hq - 1])])
    _check_rows(w, qkv, out, lse, bhr, f"{w.name} 1024 rows per head + boundary rows")


def test_special_zero_query_and_zero_scale(ra):
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(1, 2, 1, 640, 128, seed=11)
    zq = torch.zeros_like(q)
    # Q = 0: every allowed key equally likely -> prefix means, lse = ln(r + 1)
    out, lse = run(ra, zq, k, v, 5, True, 1.0 / math.sqrt(128))
    vv = to_np(v)[0, :, 0, :]
    pref = np.cumsum(vv, axis=0) / np.arange(1, 641)[:, None]
    compare(out[0, :, 0, :], lse[0, 0], pref, np.log(np.arange(1, 641)), "q=0")
    # scale = 0 gives the same uniform weights for any q
    out2, lse2 = run(ra, q, k, v, 5, True, 0.0)
    compare(out2[0, :, 1, :], lse2[0, 1], pref, np.log(np.arange(1, 641)), "scale=0")


def test_special_causal_row0_and_constant_values(ra):
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(1, 2, 2, 512, 64, seed=12)
    out, lse = run(ra, q, k, v, 4, True)
    # causal row 0 of every ring block's first host sees key 0 only
    np.testing.assert_array_equal(to_np(out[0, 0]), to_np(v[0, 0]))
    # constant V reproduces V
    cv = v[:, :1].expand_as(v).contiguous()
    out2, _ = run(ra, q, k, cv, 4, False)
    err = np.abs(to_np(out2) - to_np(cv)).max()
    assert err <= 1e-2, err


def test_deterministic_and_schedule_invariant(ra):
    """The result does not depend on how many persistent CTAs share the work
    or in which order they take the units (each unit is computed the same way
    whichever CTA takes it, whenever)."""
    from ring_attention_ordered_b200 import _lib
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(2, 4, 2, 1024, 128, seed=13)
    ref = run(ra, q, k, v, 4, True)
    try:
        for sched in (_lib.RA_SCHEDULE_LONGEST_FIRST, _lib.RA_SCHEDULE_HEAD_MAJOR):
            _lib.ring_attn_set_schedule(sched)
            for cap in (1, 3, 7, 0):
                _lib.ring_attn_set_max_ctas(cap)
                got = run(ra, q, k, v, 4, True)
                assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1]), (sched, cap)
    finally:
        _lib.ring_attn_set_max_ctas(0)
        _lib.ring_attn_set_schedule(_lib.RA_SCHEDULE_AUTO)


def test_bounded_wait_reports_timeout_and_recovers(ra):
    """A load that never comes makes the first bounded wait run out: the call
    reports RA_ERR_TIMEOUT, the context stays usable and the next call is
    correct (the aborted CTAs released their tensor memory)."""
    from ring_attention_ordered_b200 import _lib
    from ring_attention_ordered_b200.inputs import make_inputs
    q, k, v = make_inputs(1, 2, 2, 512, 128, seed=14)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    try:
        _lib.ring_attn_set_wait_limit_ns(200_000_000)
        _lib.ring_attn_debug_inject(1)
        ra.fwd(qd, kd, vd, 4, True)
        with pytest.raises(_lib.RingAttnError) as ei:
            ra.check_status()
        assert ei.value.status == _lib.RA_ERR_TIMEOUT
    finally:
        _lib.ring_attn_debug_inject(0)
        _lib.ring_attn_set_wait_limit_ns(0)
    full_compare(ra, q, k, v, 4, True, what="after timeout")


def test_invalid_arguments_on_device(ra):
    from ring_attention_ordered_b200 import _lib
    q = torch.zeros((1, 256, 2, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((1, 2, 256), dtype=torch.float32, device="cuda")
    p = q.data_ptr()
    with pytest.raises(_lib.RingAttnError) as ei:   # misaligned q
        _lib.ring_attn_fwd(p + 2, p, p, out.data_ptr(), lse.data_ptr(), 1, 2, 2, 256, 128, 2, 1,
                           0.1, 0)
    assert ei.value.status == _lib.RA_ERR_INVALID_ARG
    with pytest.raises(_lib.RingAttnError) as ei:   # output overlaps an input
        _lib.ring_attn_fwd(p, p, p, p, lse.data_ptr(), 1, 2, 2, 256, 128, 2, 1, 0.1, 0)
    assert ei.value.status == _lib.RA_ERR_INVALID_ARG


def test_work_queue_concurrent_streams_and_graph_replay(ra):
    """The forward kernels take units from a per-launch queue counter (one of
    a ring of device counters, zeroed by a stream-ordered memset).  Launches
    on two streams at once, and a forward captured in a CUDA graph and
    replayed, must give bitwise the results of plain launches."""
    from ring_attention_ordered_b200.inputs import make_inputs
    cases = [make_inputs(1, 8, 2, 4096, 128, seed=61), make_inputs(2, 4, 4, 2048, 128, seed=62)]
    dev = [tuple(t.cuda() for t in c) for c in cases]
    ref = [ra.fwd(q, k, v, 4, True) for q, k, v in dev]
    torch.cuda.synchronize()
    # concurrent: both problems in flight on their own streams, three times
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        for (q, k, v), s in zip(dev, streams):
            outs.append(ra.fwd(q, k, v, 4, True, stream=s))
    for s in streams:
        s.synchronize()
    ra.check_status()
    for i, (o, l_) in enumerate(outs):
        assert torch.equal(o, ref[i % 2][0]) and torch.equal(l_, ref[i % 2][1])
    # graph: the counter reset is captured with the launch, so replays work
    q, k, v = dev[0]
    out = torch.empty_like(q)
    lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float32, device="cuda")
    ra.fwd(q, k, v, 4, True, out=out, lse=lse)          # first call outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ra.fwd(q, k, v, 4, True, out=out, lse=lse, stream=torch.cuda.current_stream())
    for _ in range(3):
        out.zero_()
        lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        ra.check_status()
        assert torch.equal(out, ref[0][0]) and torch.equal(lse, ref[0][1])
    del g
