"""Ring attention across processes: the method's own sharding of the sequence.

"Ring Attention 环注意力" (L3 definition, L4 §4.2): N hosts form a ring.  Host
i holds its query rows and, at ring step t, the K/V rows of host
j = (i - t) mod N.  Each step it runs exact blockwise attention against the
K/V block in hand, folds the partial result into its running output, and
passes the K/V block on to host i + 1 while it receives the next one from
host i - 1; after N steps its output is exact attention over the whole
sequence.  The transfer of step t runs while step t computes (L4 §4.5
limitation 1, L5 pitfall 4: asynchronous exchange overlapped with compute).

Layouts of the sequence over the hosts (which rows host i holds), as chunks:

``contiguous``
    rows [i*l, (i+1)*l): the pages' layout, one chunk per host.  Causal: the
    host's own block is diagonal-masked, earlier blocks are full, later ones
    are skipped, so host N-1 computes N visits and host 0 one (L4 §4.5
    limitation 2: the others wait, yet still pass K/V on).
``zigzag``
    the sequence cut into 2N chunks of l/2 rows; host i holds chunks i and
    2N-1-i (the "Zigzag Ring" the pages name as the fix for limitation 2).
    Causal: every host computes the same amount at every step.
``striped``
    host i holds rows i, i+N, i+2N, ... (the interleaved sharding of
    "Striped Attention", L4 §4.8).  Causal: every visit is triangular: the
    keys of hosts j <= i up to the query's own local row, those of hosts j > i
    strictly before it.

Host tensors are chunk-major: q [C, B, c, Hq, d], k/v [C, B, c, Hkv, d]
(C = 2 chunks for zigzag, else 1; c rows per chunk); ``shard``/``unshard``
convert from and to the whole sequence [B, L, H, d].  Every visit is one
``ring_attn_fwd_visit`` launch on a (query chunk, K/V chunk) pair, which folds
into the fp32 accumulator in its epilogue.  The exchange uses
torch.distributed point-to-point ops (NCCL between GPUs, gloo between CPU
processes).  There is no other compute path: without the CUDA library the
default visit raises.

The backward pass (``ring_attention_bwd``) walks the same plan: each step a
host adds its query block's dQ share (``ring_attn_bwd_visit``, dQ half) and
then its share of the held block's dK, dV to fp32 accumulators that travel
with the K/V block; one extra hop after the last step brings every block's
accumulators home, where ``ring_attn_round_bf16`` rounds them.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch
import torch.distributed as dist

LAYOUTS = ("contiguous", "zigzag", "striped")

FULL, DIAG, STRICT = 0, 1, 2   # visit masks (the `diag` argument of the visit call)


def n_chunks(layout: str) -> int:
    if layout not in LAYOUTS:
        raise ValueError(f"unknown layout {layout!r} (one of {LAYOUTS})")
    return 2 if layout == "zigzag" else 1


def chunk_ids(host: int, world: int, layout: str) -> list[int]:
    """Sequence chunks a host holds, in its local order (contiguous: block
    `host` of N; zigzag: chunks `host` and 2N-1-`host` of 2N; striped: the
    host's stripe, one chunk)."""
    if n_chunks(layout) == 2:
        return [host, 2 * world - 1 - host]
    return [host]


@dataclass(frozen=True)
class Visit:
    qc: int     # index of the query chunk on this host
    kc: int     # index of the K/V chunk in the block held at this step
    mask: int   # FULL, DIAG (keys c <= r) or STRICT (keys c < r), local rows


def visit_plan(host: int, world: int, causal: bool, layout: str):
    """For each ring step t = 0..N-1: (j, visits), j = (host - t) mod N the
    host whose K/V block is held, visits the chunk pairs to compute (pairs
    that the causal mask empties entirely are left out)."""
    if world < 1 or not 0 <= host < world:
        raise ValueError(f"host {host} outside a ring of {world}")
    plan = []
    for t in range(world):
        j = (host - t) % world
        visits = []
        if layout == "striped":
            # global row of local row r on host h is r*N + h: key (c, j) is
            # allowed for query (r, host) iff c*N + j <= r*N + host
            mask = FULL if not causal else (DIAG if j <= host else STRICT)
            visits.append(Visit(0, 0, mask))
        else:
            for qc, a in enumerate(chunk_ids(host, world, layout)):
                for kc, b in enumerate(chunk_ids(j, world, layout)):
                    if not causal or b < a:
                        visits.append(Visit(qc, kc, FULL))
                    elif b == a:
                        visits.append(Visit(qc, kc, DIAG))
        plan.append((j, visits))
    return plan


def visit_work(mask: int) -> float:
    """Work of one visit in units of a full chunk pair (a triangle is half)."""
    return 1.0 if mask == FULL else 0.5


# ------------------------------------------------------------------ layouts

def shard(x: torch.Tensor, host: int, world: int, layout: str) -> torch.Tensor:
    """The rows host `host` holds, chunk-major: x [B, L, H, d] ->
    [C, B, c, H, d] (a copy)."""
    B, L, H, d = x.shape
    C = n_chunks(layout)
    if L % (C * world) != 0:
        raise ValueError(f"L={L} does not split into {C * world} equal chunks")
    if layout == "striped":
        return x[:, host::world].unsqueeze(0).contiguous()
    c = L // (C * world)
    parts = [x[:, g * c:(g + 1) * c] for g in chunk_ids(host, world, layout)]
    return torch.stack(parts, 0).contiguous()


def unshard(parts, layout: str) -> torch.Tensor:
    """Inverse of ``shard``: the hosts' chunk-major row sets [C, B, c, H, d]
    (list in host order) -> [B, L, H, d]."""
    world = len(parts)
    C, B, c, H, d = parts[0].shape
    out = parts[0].new_empty((B, C * c * world, H, d))
    for host, p in enumerate(parts):
        if layout == "striped":
            out[:, host::world] = p[0]
        else:
            for i, g in enumerate(chunk_ids(host, world, layout)):
                out[:, g * c:(g + 1) * c] = p[i]
    return out


def unshard_lse(parts, layout: str) -> torch.Tensor:
    """``unshard`` for lse: [C, B, H, c] per host -> [B, H, L]."""
    world = len(parts)
    C, B, H, c = parts[0].shape
    out = parts[0].new_empty((B, H, C * c * world))
    for host, p in enumerate(parts):
        if layout == "striped":
            out[:, :, host::world] = p[0]
        else:
            for i, g in enumerate(chunk_ids(host, world, layout)):
                out[:, :, g * c:(g + 1) * c] = p[i]
    return out


# ------------------------------------------------------------------ visits

def cuda_visit(q, k, v, o_acc, lse_acc, mask, fold, scale, out):
    """One chunk-pair visit through the C ABI (ring_attn_fwd_visit)."""
    from . import api
    api.fwd_visit(q, k, v, o_acc, lse_acc, mask, fold, scale, out)


def _run_host(q, k_blocks, v_blocks, plan, scale, visit, exchange_step=None):
    """Run one host's plan.  k_blocks(t)/v_blocks(t) give the K/V block held
    at step t ([C, B, c, Hkv, d]); ``exchange_step(t)`` (if given) starts the
    transfer of step t and returns a callable that waits for it."""
    C, B, c, Hq, d = q.shape
    o_acc = torch.empty((C, B, c, Hq, d), dtype=torch.float32, device=q.device)
    lse_acc = torch.empty((C, B, Hq, c), dtype=torch.float32, device=q.device)
    out = torch.empty_like(q)
    last = {}
    for t, (_, visits) in enumerate(plan):
        for n, vi in enumerate(visits):
            last[vi.qc] = (t, n)
    if len(last) != C:
        raise RuntimeError("a query chunk receives no visit")
    started = set()
    for t, (_, visits) in enumerate(plan):
        wait = exchange_step(t) if exchange_step is not None else None
        kb, vb = k_blocks(t), v_blocks(t)
        for n, vi in enumerate(visits):
            fold = vi.qc in started
            started.add(vi.qc)
            visit(q[vi.qc], kb[vi.kc], vb[vi.kc], o_acc[vi.qc], lse_acc[vi.qc], vi.mask, fold,
                  scale, out[vi.qc] if last[vi.qc] == (t, n) else None)
        if wait is not None:
            wait()
    return out, lse_acc


class P2PRing:
    """K/V exchange between ring neighbours over a torch.distributed group:
    send the held block to host i+1, receive the next from host i-1."""

    def __init__(self, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        nxt, prv = (self.rank + 1) % self.world, (self.rank - 1) % self.world
        if group is None:
            self.next, self.prev = nxt, prv
        else:
            self.next = dist.get_global_rank(group, nxt)
            self.prev = dist.get_global_rank(group, prv)

    def start(self, send, recv):
        ops = [dist.P2POp(dist.isend, s, self.next, self.group) for s in send]
        ops += [dist.P2POp(dist.irecv, r, self.prev, self.group) for r in recv]
        works = dist.batch_isend_irecv(ops)

        def wait():
            for w in works:
                w.wait()
        return wait


def ring_attention(q, k, v, causal: bool, scale: float | None = None, layout: str = "contiguous",
                   group=None, visit=None):
    """This process's share of ring attention over a torch.distributed group
    (one process per host, ranks in ring order).

    q [C, B, c, Hq, d], k/v [C, B, c, Hkv, d]: this host's rows in the
    layout's chunk-major form (``shard``); a 4-d [B, l, H, d] block is taken
    as C = 1.  Returns (out [C, B, c, Hq, d] in q's dtype, lse fp32
    [C, B, Hq, c]), 4-d / 3-d again for a 4-d q.  ``visit`` replaces the CUDA
    visit (tests on CPU processes).  K/V blocks are double-buffered: the
    receive of step t+1's block overlaps step t's visits.
    """
    squeeze = q.dim() == 4
    if squeeze:
        q, k, v = q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
    if q.shape[0] != n_chunks(layout):
        raise ValueError(f"layout {layout} wants {n_chunks(layout)} chunks, got {q.shape[0]}")
    ring = P2PRing(group)
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    plan = visit_plan(ring.rank, ring.world, causal, layout)
    held = [(k, v)]
    spare = []

    def exchange_step(t):
        if t == ring.world - 1:
            return None
        cur_k, cur_v = held[t]
        if len(spare) < 2:
            spare.append((torch.empty_like(k), torch.empty_like(v)))
        nk, nv = spare[t % 2]
        held.append((nk, nv))
        return ring.start([cur_k, cur_v], [nk, nv])

    out, lse = _run_host(q, lambda t: held[t][0], lambda t: held[t][1], plan, scale,
                         visit or cuda_visit, exchange_step)
    if squeeze:
        return out[0], lse[0]
    return out, lse


def ring_attention_emulated(q, k, v, world: int, causal: bool, scale: float | None = None,
                            layout: str = "contiguous", visit=None, hosts=None):
    """All hosts of a ring of ``world`` on one device: q [B, L, Hq, d],
    k/v [B, L, Hkv, d] (the whole sequence).  Each host runs exactly the
    visits and folds of ``ring_attention``, with the K/V block of every step
    taken from the whole tensors instead of received.  Returns the whole
    (out [B, L, Hq, d], lse [B, Hq, L]).  ``hosts`` restricts the run to some
    hosts (their rows only are written; the rest stay uninitialised)."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    ks = [shard(k, h, world, layout) for h in range(world)]
    vs = [shard(v, h, world, layout) for h in range(world)]
    outs, lses = [], []
    for host in range(world):
        qh = shard(q, host, world, layout)
        if hosts is not None and host not in hosts:
            outs.append(torch.empty_like(qh))
            lses.append(torch.empty((qh.shape[0], qh.shape[1], qh.shape[3], qh.shape[2]),
                                    dtype=torch.float32, device=q.device))
            continue
        plan = visit_plan(host, world, causal, layout)
        o, l = _run_host(qh, lambda t: ks[plan[t][0]], lambda t: vs[plan[t][0]], plan, scale,
                         visit or cuda_visit)
        outs.append(o)
        lses.append(l)
    return unshard(outs, layout), unshard_lse(lses, layout)


# ------------------------------------------------------------------ backward

def cuda_bwd_visit(q, k, v, out, dout, lse, ws, mask, parts, dq_acc, dk_acc, dv_acc, scale, dq):
    """One backward chunk-pair visit through the C ABI (ring_attn_bwd_visit);
    the accumulators start at zero and every visit adds its share."""
    from . import api
    api.bwd_visit(q, k, v, out, dout, lse, ws, mask, parts, dq_acc, dk_acc, dv_acc, True, True,
                  scale, dq)


def cuda_round(src, like):
    """A travelling fp32 gradient accumulator, home, rounded to bf16 (C ABI)."""
    from . import api
    return api.round_bf16(src)


def _last_visits(plan):
    last = {}
    for t, (_, visits) in enumerate(plan):
        for n, vi in enumerate(visits):
            last[vi.qc] = (t, n)
    return last


def _bwd_phase(part, t, visits, last_q, q, out, dout, lse, ws, kb, vb, dq_acc, dq, dk_acc, dv_acc,
               scale, visit):
    for n, vi in enumerate(visits):
        if part == 1:
            visit(q[vi.qc], kb[vi.kc], vb[vi.kc], out[vi.qc], dout[vi.qc], lse[vi.qc], ws[vi.qc],
                  vi.mask, 1, dq_acc[vi.qc], None, None, scale,
                  dq[vi.qc] if last_q[vi.qc] == (t, n) else None)
        else:
            visit(q[vi.qc], kb[vi.kc], vb[vi.kc], out[vi.qc], dout[vi.qc], lse[vi.qc], ws[vi.qc],
                  vi.mask, 2, None, dk_acc[vi.kc], dv_acc[vi.kc], scale, None)


def _workspaces(q):
    C, B, c, Hq, _ = q.shape
    return [torch.empty(max(16, B * Hq * c * 4), dtype=torch.uint8, device=q.device)
            for _ in range(C)]


def ring_attention_bwd(q, k, v, out, dout, lse, causal: bool, scale: float | None = None,
                       layout: str = "contiguous", group=None, visit=None, finish=None):
    """This process's share of the ring attention backward pass over a
    torch.distributed group.

    q, out, dout [C, B, c, Hq, d], k, v [C, B, c, Hkv, d] and lse
    [C, B, Hq, c] are this host's rows (``shard``; ``out`` and ``lse`` as
    ``ring_attention`` returned them, 4-d / 3-d for C = 1).  Every ring step
    the host computes its query block's dQ share against the K/V block it
    holds, then adds its dK, dV share to that block's fp32 accumulators, which
    travel around the ring with K and V (received from host i-1, passed to
    host i+1); after the last step one more hop brings each block's
    accumulators home, where they are rounded to bf16.  The K/V transfer of
    step t+1 overlaps step t; the accumulators of a step are received while
    the dQ half of the step computes.  Returns (dq, dk, dv) in the layout of
    q, k, v.  ``visit``/``finish`` replace the CUDA visit and rounding
    (tests on CPU processes)."""
    squeeze = q.dim() == 4
    if squeeze:
        q, k, v, out, dout = (x.unsqueeze(0) for x in (q, k, v, out, dout))
        lse = lse.unsqueeze(0)
    visit = visit or cuda_bwd_visit
    finish = finish or cuda_round
    ring = P2PRing(group)
    N = ring.world
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    plan = visit_plan(ring.rank, N, causal, layout)
    last_q = _last_visits(plan)
    dq_acc = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    dq = torch.empty_like(q)
    ws = _workspaces(q)
    acc = [(torch.zeros(k.shape, dtype=torch.float32, device=k.device),
            torch.zeros(v.shape, dtype=torch.float32, device=v.device)),
           (torch.empty(k.shape, dtype=torch.float32, device=k.device),
            torch.empty(v.shape, dtype=torch.float32, device=v.device))]
    held = [(k, v)]
    spare = []
    acc_wait = None
    for t, (_, visits) in enumerate(plan):
        kv_wait = None
        if t < N - 1:
            if len(spare) < 2:
                spare.append((torch.empty_like(k), torch.empty_like(v)))
            nk, nv = spare[t % 2]
            kv_wait = ring.start(list(held[t]), [nk, nv])
            held.append((nk, nv))
        kb, vb = held[t]
        dka, dva = acc[t % 2]
        _bwd_phase(1, t, visits, last_q, q, out, dout, lse, ws, kb, vb, dq_acc, dq, dka, dva,
                   scale, visit)
        if acc_wait is not None:
            acc_wait()          # this block's accumulators, from host i-1
        _bwd_phase(2, t, visits, last_q, q, out, dout, lse, ws, kb, vb, dq_acc, dq, dka, dva,
                   scale, visit)
        if N > 1:
            acc_wait = ring.start([dka, dva], list(acc[(t + 1) % 2]))
        if kv_wait is not None:
            kv_wait()
    if acc_wait is not None:
        acc_wait()              # this host's own block, home after N hops
    fk, fv = acc[N % 2] if N > 1 else acc[0]
    dk, dv = finish(fk, k), finish(fv, v)
    if squeeze:
        return dq[0], dk[0], dv[0]
    return dq, dk, dv


def ring_attention_bwd_emulated(q, k, v, out, dout, lse, world: int, causal: bool,
                                scale: float | None = None, layout: str = "contiguous",
                                visit=None, finish=None):
    """All hosts of ``ring_attention_bwd`` on one device, whole-sequence
    tensors in (q, out, dout [B, L, Hq, d], k, v [B, L, Hkv, d], lse
    [B, Hq, L]) and out: every host runs exactly its visits, each K/V block's
    accumulators receive the hosts' shares in the ring's order (host j at
    step 0, j+1 at step 1, ...), without the exchange."""
    visit = visit or cuda_bwd_visit
    finish = finish or cuda_round
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    sh = lambda x, h: shard(x, h, world, layout)  # noqa: E731
    lse_rows = lse.permute(0, 2, 1).unsqueeze(-1)          # [B, L, Hq, 1]
    hosts = []
    for h in range(world):
        qh = sh(q, h)
        hosts.append(dict(
            q=qh, out=sh(out, h), dout=sh(dout, h),
            lse=sh(lse_rows, h)[..., 0].permute(0, 1, 3, 2).contiguous(),
            k=sh(k, h), v=sh(v, h), ws=_workspaces(qh),
            dq_acc=torch.zeros(qh.shape, dtype=torch.float32, device=q.device),
            dq=torch.empty_like(qh), plan=visit_plan(h, world, causal, layout)))
    for hd in hosts:
        hd["last_q"] = _last_visits(hd["plan"])
    acc = [(torch.zeros(hd["k"].shape, dtype=torch.float32, device=k.device),
            torch.zeros(hd["v"].shape, dtype=torch.float32, device=v.device)) for hd in hosts]
    for t in range(world):
        for part in (1, 2):
            for hd in hosts:
                j, visits = hd["plan"][t]
                kb, vb = hosts[j]["k"], hosts[j]["v"]
                _bwd_phase(part, t, visits, hd["last_q"], hd["q"], hd["out"], hd["dout"],
                           hd["lse"], hd["ws"], kb, vb, hd["dq_acc"], hd["dq"], acc[j][0],
                           acc[j][1], scale, visit)
    dq = unshard([hd["dq"] for hd in hosts], layout)
    dk = unshard([finish(acc[h][0], hosts[h]["k"]) for h in range(world)], layout)
    dv = unshard([finish(acc[h][1], hosts[h]["v"]) for h in range(world)], layout)
    return dq, dk, dv


class RingAttentionFn(torch.autograd.Function):
    """Autograd bridge for the multi-process ring: forward by
    ``ring_attention``, backward by ``ring_attention_bwd`` (same layout,
    group and visits)."""

    @staticmethod
    def forward(ctx, q, k, v, causal, scale, layout, group, visit, bwd_visit, finish):
        out, lse = ring_attention(q, k, v, causal, scale, layout, group, visit)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.args = (causal, scale, layout, group, bwd_visit, finish)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        causal, scale, layout, group, bwd_visit, finish = ctx.args
        dq, dk, dv = ring_attention_bwd(q, k, v, out, dout.contiguous().to(out.dtype), lse,
                                        causal, scale, layout, group, bwd_visit, finish)
        return dq, dk, dv, None, None, None, None, None, None, None


def ring_attention_fn(q, k, v, causal: bool, scale: float | None = None,
                      layout: str = "contiguous", group=None, visit=None, bwd_visit=None,
                      finish=None):
    """Differentiable ``ring_attention``: this host's output, with gradients
    for its q, k and v through the backward ring."""
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    return RingAttentionFn.apply(q, k, v, causal, scale, layout, group, visit, bwd_visit, finish)
