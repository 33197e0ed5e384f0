"""Host logic of the multi-process ring (ring_attention_ordered_b200.ring) on
the CPU: the visit plans of the three layouts, their coverage of the causal
mask, the balance the zigzag and striped layouts buy, the layout shuffles,
and the ring itself over gloo processes with the fp64 oracle standing in for
the CUDA visit (the exchange, the double buffering and the fold order are
what is under test; the visit kernel is tested on the GPU)."""

from __future__ import annotations

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from ring_attention_ordered_b200 import ring
from ring_attention_ordered_b200.ring import DIAG, FULL, STRICT

KIND = {FULL: "full", DIAG: "masked", STRICT: "strict"}


def oracle_visit(q, k, v, o_acc, lse_acc, mask, fold, scale, out):
    """The visit contract of ring_attn_fwd_visit, computed by the oracle:
    block attention of the chunk pair, merged into (o_acc, lse_acc) when
    fold, the result rounded into out when given."""
    o_t, l_t = oracle.block_attention(q, k, v, scale, KIND[mask])
    l_t = l_t.transpose(0, 2, 1)                       # [B, c, Hq] like o's rows
    if fold:
        l_prev = lse_acc.double().numpy().transpose(0, 2, 1)
        o_t, l_t = oracle.merge(o_acc.double().numpy(), l_prev, o_t, l_t)
    o_acc.copy_(torch.from_numpy(np.ascontiguousarray(o_t)))
    lse_acc.copy_(torch.from_numpy(np.ascontiguousarray(l_t.transpose(0, 2, 1))))
    if out is not None:
        out.copy_(o_acc.to(out.dtype))


def global_rows(host, world, layout, c):
    """Global sequence row of each local row (chunk-major) of a host."""
    if layout == "striped":
        return [np.arange(c) * world + host]
    return [np.arange(c) + g * c for g in ring.chunk_ids(host, world, layout)]


# ------------------------------------------------------------------ plans

@pytest.mark.parametrize("world", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_contiguous_plan_is_the_pages_ring(world, causal):
    """The contiguous layout visits blocks (i - t) mod N in ring order with
    the oracle's causal classification (skip j > i, mask j == i)."""
    for host in range(world):
        plan = ring.visit_plan(host, world, causal, "contiguous")
        assert [j for j, _ in plan] == oracle.ring_order(host, world)
        got = [(t, j, KIND[vs[0].mask]) for t, (j, vs) in enumerate(plan) if vs]
        assert got == oracle.ring_visits(host, world, causal)


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("world", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_plans_cover_the_mask_exactly_once(layout, world, causal):
    """Over all hosts and steps, every (query row, key row) pair the mask
    allows is computed exactly once and no other pair is (brute force over
    global row numbers, 3 rows per chunk)."""
    c = 3
    L = c * ring.n_chunks(layout) * world
    count = np.zeros((L, L), dtype=np.int64)
    for host in range(world):
        qrows = global_rows(host, world, layout, c)
        for j, visits in ring.visit_plan(host, world, causal, layout):
            krows = global_rows(j, world, layout, c)
            for vi in visits:
                r, cc = np.meshgrid(np.arange(c), np.arange(c), indexing="ij")
                keep = {FULL: np.ones_like(r, bool), DIAG: cc <= r, STRICT: cc < r}[vi.mask]
                gq = qrows[vi.qc][r[keep]]
                gk = krows[vi.kc][cc[keep]]
                np.add.at(count, (gq, gk), 1)
    want = np.tril(np.ones((L, L), np.int64)) if causal else np.ones((L, L), np.int64)
    np.testing.assert_array_equal(count, want)


@pytest.mark.parametrize("layout", ["zigzag", "striped"])
@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_balanced_layouts_give_every_host_equal_work_each_step(layout, world):
    """The fix for the causal waste the pages name (L4 §4.5 limitation 2):
    under causal masking the zigzag and striped layouts give every host the
    same work at every ring step; the contiguous layout gives host i
    i + 1 of N visits."""
    work = np.array([[sum(ring.visit_work(v.mask) for v in vs)
                      for _, vs in ring.visit_plan(h, world, True, layout)]
                     for h in range(world)])
    assert np.all(work == work[0, 0])
    cont = [sum(1 for _, vs in ring.visit_plan(h, world, True, "contiguous") if vs)
            for h in range(world)]
    assert cont == list(range(1, world + 1))


@pytest.mark.parametrize("layout", ring.LAYOUTS)
def test_shard_unshard_round_trip(layout):
    x = torch.arange(2 * 24 * 3 * 2, dtype=torch.float32).reshape(2, 24, 3, 2)
    parts = [ring.shard(x, h, 3, layout) for h in range(3)]
    assert torch.equal(ring.unshard(parts, layout), x)
    lse = torch.arange(2 * 3 * 24, dtype=torch.float32).reshape(2, 3, 24)
    lparts = [ring.shard(lse.permute(0, 2, 1).unsqueeze(-1), h, 3, layout)[..., 0]
              .permute(0, 1, 3, 2) for h in range(3)]
    assert torch.equal(ring.unshard_lse(lparts, layout), lse)


def test_plan_rejects_bad_arguments():
    with pytest.raises(ValueError):
        ring.visit_plan(3, 3, True, "contiguous")
    with pytest.raises(ValueError):
        ring.n_chunks("diagonal")
    with pytest.raises(ValueError):
        ring.shard(torch.zeros(1, 10, 1, 1), 0, 3, "contiguous")


# ------------------------------------------------------------ emulated ring

def small_inputs(B=1, L=24, Hq=4, Hkv=2, d=8, seed=5):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((B, L, Hq, d), generator=g), torch.randn((B, L, Hkv, d), generator=g),
            torch.randn((B, L, Hkv, d), generator=g))


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_ring_with_oracle_visits_is_exact_attention(layout, world, causal):
    q, k, v = small_inputs()
    out, lse = ring.ring_attention_emulated(q, k, v, world, causal, 0.4, layout,
                                            visit=oracle_visit)
    o_ref, l_ref = oracle.attention(q, k, v, causal, 0.4)
    np.testing.assert_allclose(out.numpy(), o_ref, rtol=0, atol=1e-5)
    np.testing.assert_allclose(lse.numpy(), l_ref, rtol=0, atol=1e-5)


# ------------------------------------------------------------ gloo processes

def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ring_rank(rank, world, port, layout, causal, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = small_inputs(B=2, L=8 * world * ring.n_chunks(layout))
        qs, ks, vs = (ring.shard(x, rank, world, layout) for x in (q, k, v))
        k0, v0 = ks.clone(), vs.clone()
        out, lse = ring.ring_attention(qs, ks, vs, causal, 0.3, layout, visit=oracle_visit)
        # the caller's own K/V block is passed on, never overwritten
        assert torch.equal(ks, k0) and torch.equal(vs, v0)
        results[rank] = (out, lse)
    finally:
        dist.destroy_process_group()


def _spawn(target, world, *args):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=target, args=(r, world, port, *args, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
        codes = [p.exitcode for p in procs]
        return codes, dict(results)


@pytest.mark.parametrize("world,layout,causal", [
    (2, "contiguous", True), (3, "contiguous", False), (4, "contiguous", True),
    (3, "zigzag", True), (4, "zigzag", True), (2, "striped", True), (4, "striped", False),
])
def test_gloo_ring_is_exact_attention(world, layout, causal):
    codes, res = _spawn(_ring_rank, world, layout, causal)
    assert codes == [0] * world, codes
    out = ring.unshard([res[r][0] for r in range(world)], layout)
    lse = ring.unshard_lse([res[r][1] for r in range(world)], layout)
    q, k, v = small_inputs(B=2, L=8 * world * ring.n_chunks(layout))
    o_ref, l_ref = oracle.attention(q, k, v, causal, 0.3)
    np.testing.assert_allclose(out.numpy(), o_ref, rtol=0, atol=1e-5)
    np.testing.assert_allclose(lse.numpy(), l_ref, rtol=0, atol=1e-5)


def _dying_rank(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        os._exit(3)           # the neighbour dies before the first exchange
    q, k, v = small_inputs(L=16)
    try:
        ring.ring_attention(q, k, v, True, 0.3, visit=oracle_visit)
        results[rank] = "returned"
    except Exception as e:  # noqa: BLE001 - any error ends the wait
        results[rank] = f"raised {type(e).__name__}"


def test_a_dead_neighbour_ends_the_ring_with_an_error():
    """A host that dies before its exchange: the survivor's receive fails
    (connection closed, or the group's 10 s timeout) instead of waiting for
    ever."""
    codes, res = _spawn(_dying_rank, 2)
    assert codes[1] == 3
    assert res.get(0, "").startswith("raised"), res


# ------------------------------------------------------------------ backward

def oracle_bwd_visit(q, k, v, out, dout, lse, ws, mask, parts, dq_acc, dk_acc, dv_acc, scale, dq):
    """The contract of ring_attn_bwd_visit (accumulators add the visit's
    share), computed by the oracle's block_attention_bwd."""
    pq, pk, pv = oracle.block_attention_bwd(q, k, v, out, dout, lse, scale, KIND[mask])
    if parts & 1:
        dq_acc += torch.from_numpy(pq).to(dq_acc.dtype)
        if dq is not None:
            dq.copy_(dq_acc.to(dq.dtype))
    if parts & 2:
        dk_acc += torch.from_numpy(pk).to(dk_acc.dtype)
        dv_acc += torch.from_numpy(pv).to(dv_acc.dtype)


def plain_finish(src, like):
    return src.to(like.dtype)


def bwd_inputs(B, L, Hq=4, Hkv=2, d=8, seed=8, causal=True, scale=0.3):
    q, k, v = small_inputs(B=B, L=L, Hq=Hq, Hkv=Hkv, d=d, seed=seed)
    g = torch.Generator().manual_seed(seed + 1)
    do = torch.randn((B, L, Hq, d), generator=g)
    out, lse = oracle.attention(q, k, v, causal, scale)
    return q, k, v, do, torch.from_numpy(out).float(), torch.from_numpy(lse).float()


@pytest.mark.parametrize("layout", ring.LAYOUTS)
@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_ring_bwd_with_oracle_visits_is_the_gradient(layout, world, causal):
    q, k, v, do, out, lse = bwd_inputs(1, 24, causal=causal)
    got = ring.ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal, 0.3, layout,
                                           visit=oracle_bwd_visit, finish=plain_finish)
    want = oracle.attention_bwd(q, k, v, do, causal, 0.3)
    for g_, w_ in zip(got, want):
        np.testing.assert_allclose(g_.numpy(), w_, rtol=0, atol=2e-5)


def _ring_bwd_rank(rank, world, port, layout, causal, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        L = 8 * world * ring.n_chunks(layout)
        q, k, v, do, out, lse = bwd_inputs(2, L, causal=causal)
        sh = lambda x: ring.shard(x, rank, world, layout)  # noqa: E731
        lse_h = sh(lse.permute(0, 2, 1).unsqueeze(-1))[..., 0].permute(0, 1, 3, 2).contiguous()
        ks, vs = sh(k), sh(v)
        k0, v0 = ks.clone(), vs.clone()
        grads = ring.ring_attention_bwd(sh(q), ks, vs, sh(out), sh(do), lse_h, causal, 0.3, layout,
                                        visit=oracle_bwd_visit, finish=plain_finish)
        assert torch.equal(ks, k0) and torch.equal(vs, v0)
        results[rank] = grads
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout,causal", [
    (2, "contiguous", True), (3, "contiguous", False), (4, "zigzag", True), (3, "striped", True),
])
def test_gloo_ring_bwd_is_the_gradient(world, layout, causal):
    """dK and dV accumulators travel the ring with their K/V block between
    gloo processes and come home after N hops."""
    codes, res = _spawn(_ring_bwd_rank, world, layout, causal)
    assert codes == [0] * world, codes
    L = 8 * world * ring.n_chunks(layout)
    q, k, v, do, out, lse = bwd_inputs(2, L, causal=causal)
    want = oracle.attention_bwd(q, k, v, do, causal, 0.3)
    for i in range(3):
        got = ring.unshard([res[r][i] for r in range(world)], layout)
        np.testing.assert_allclose(got.numpy(), want[i], rtol=0, atol=2e-5)


def _autograd_rank(rank, world, port, layout, causal, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        L = 8 * world * ring.n_chunks(layout)
        q, k, v = small_inputs(B=1, L=L, seed=11)
        g = torch.Generator().manual_seed(12)
        do = torch.randn(q.shape, generator=g)
        sh = lambda x: ring.shard(x, rank, world, layout)  # noqa: E731
        qs, ks, vs = (sh(x).requires_grad_() for x in (q, k, v))
        out = ring.ring_attention_fn(qs, ks, vs, causal, 0.35, layout, visit=oracle_visit,
                                     bwd_visit=oracle_bwd_visit, finish=plain_finish)
        (out * sh(do)).sum().backward()
        results[rank] = (out.detach(), qs.grad, ks.grad, vs.grad)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "zigzag"), (3, "striped")])
def test_gloo_ring_autograd_matches_the_oracle(world, layout):
    """ring_attention_fn through torch.autograd on gloo processes: the
    outputs and the q, k, v gradients of every host equal the oracle's."""
    codes, res = _spawn(_autograd_rank, world, layout, True)
    assert codes == [0] * world, codes
    L = 8 * world * ring.n_chunks(layout)
    q, k, v = small_inputs(B=1, L=L, seed=11)
    g = torch.Generator().manual_seed(12)
    do = torch.randn(q.shape, generator=g)
    o_ref, _ = oracle.attention(q, k, v, True, 0.35)
    g_ref = oracle.attention_bwd(q, k, v, do, True, 0.35)
    got = [ring.unshard([res[r][i] for r in range(world)], layout) for i in range(4)]
    np.testing.assert_allclose(got[0].numpy(), o_ref, rtol=0, atol=2e-5)
    for a, b in zip(got[1:], g_ref):
        np.testing.assert_allclose(a.numpy(), b, rtol=0, atol=2e-5)
