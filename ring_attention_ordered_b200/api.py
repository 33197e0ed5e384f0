"""Torch-facing wrapper: checks tensors, allocates outputs with torch and
passes raw pointers plus a CUDA stream (the caller's ``stream``, else the
current one) to the C ABI.  All arithmetic happens in the library's kernels.

Outputs and temporaries that a call allocates are allocated while the stream
the kernels run on is current.  torch's caching allocator ties a block to the
stream that was current at allocation and reuses it only in that stream's
order.  A temporary freed when the call returns, such as the backward's
workspace, is therefore not handed to other work before the kernels that use
it have finished.
"""

from __future__ import annotations

import math
from contextlib import contextmanager

import torch

from . import _lib


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


@contextmanager
def _on(device, stream):
    """Make ``device`` and the call's stream current; yields the stream
    handle for the C ABI."""
    with torch.cuda.device(device):
        s = stream if stream is not None else torch.cuda.current_stream(device)
        with torch.cuda.stream(s):
            yield int(s.cuda_stream)


def _check_cuda(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def _check_out(t: torch.Tensor, name: str, dtype: torch.dtype, shape):
    """A caller-supplied output must match the shape the kernel writes: the
    library writes through raw pointers and cannot see a buffer's size."""
    _check_cuda(t, name, dtype, len(shape))
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ring: int, causal: bool,
        scale: float | None = None, out: torch.Tensor | None = None,
        lse: torch.Tensor | None = None, stream=None):
    """Ring-ordered attention forward.  q [B, L, Hq, d], k/v [B, L, Hkv, d]
    (bf16, contiguous, on the GPU).  Returns (out bf16 [B, L, Hq, d],
    lse fp32 [B, Hq, L]).  ``scale`` defaults to 1/sqrt(d)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_cuda(t, n, torch.bfloat16, 4)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} does not match q {tuple(q.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on(q.device, stream) as sh:
        if out is None:
            out = torch.empty_like(q)
        if lse is None:
            lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
        _check_out(out, "out", torch.bfloat16, (B, L, Hq, d))
        _check_out(lse, "lse", torch.float32, (B, Hq, L))
        _lib.ring_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           lse.data_ptr(), B, Hq, Hkv, L, d, n_ring, causal, scale, sh)
    return out, lse


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
        dout: torch.Tensor, lse: torch.Tensor, n_ring: int, causal: bool,
        scale: float | None = None, dq: torch.Tensor | None = None,
        dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
        workspace: torch.Tensor | None = None, stream=None):
    """Backward pass of ``fwd``: q/k/v/n_ring/causal/scale as given to it, its
    out (bf16 [B, L, Hq, d]) and lse (fp32 [B, Hq, L]), and dout (bf16, like
    out).  Returns (dq, dk, dv) in bf16.  ``workspace`` (any CUDA tensor of at
    least ``ring_attn_bwd_workspace_size`` bytes) is allocated if omitted."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check_cuda(t, n, torch.bfloat16, 4)
    _check_cuda(lse, "lse", torch.float32, 3)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} does not match q {tuple(q.shape)}")
    if out.shape != q.shape or dout.shape != q.shape or lse.shape != (B, Hq, L):
        raise ValueError("out/dout/lse shapes do not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on(q.device, stream) as sh:
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
            _check_cuda(t, n, torch.bfloat16, 4)
            if t.shape != ref.shape:
                raise ValueError(f"{n} shape does not match")
        need = _lib.ring_attn_bwd_workspace_size(B, Hq, L)
        if workspace is None:
            workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
        if not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        ws_bytes = workspace.numel() * workspace.element_size()
        _lib.ring_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                           dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                           dv.data_ptr(), workspace.data_ptr(), ws_bytes, B, Hq, Hkv, L, d,
                           n_ring, causal, scale, sh)
    return dq, dk, dv


def bwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                dout: torch.Tensor, lse: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor,
                dv: torch.Tensor, n_ring: int, causal: bool, scale: float | None = None,
                stream=None):
    """``bwd`` through ring_attn_bwd_noalloc: no workspace, results written
    into the given dq/dk/dv (bf16, shapes of q/k/v); B * Hq * L must not
    exceed 1,048,576."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"), (dq, "dq"),
                 (dk, "dk"), (dv, "dv")):
        _check_cuda(t, n, torch.bfloat16, 4)
    _check_cuda(lse, "lse", torch.float32, 3)
    B, L, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, L, Hkv, d) or v.shape != k.shape or out.shape != q.shape or \
            dout.shape != q.shape or lse.shape != (B, Hq, L):
        raise ValueError("k/v/out/dout/lse shapes do not match q")
    for t, n, ref in ((dq, "dq", q), (dk, "dk", k), (dv, "dv", v)):
        _check_out(t, n, torch.bfloat16, tuple(ref.shape))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on(q.device, stream) as sh:
        _lib.ring_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                   dv.data_ptr(), B, Hq, Hkv, L, d, n_ring, causal, scale, sh)
    return dq, dk, dv


def bwd_visit(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
              dout: torch.Tensor, lse: torch.Tensor, workspace: torch.Tensor, diag: int,
              parts: int, dq_acc: torch.Tensor | None = None, dk_acc: torch.Tensor | None = None,
              dv_acc: torch.Tensor | None = None, fold_q: bool = False, fold_kv: bool = False,
              scale: float | None = None, dq: torch.Tensor | None = None, stream=None):
    """One backward ring visit (ring_attn_bwd_visit): the host's query block
    q/out/dout [B, l, Hq, d] (bf16) with its final lse [B, Hq, l] against the
    K/V block k/v [B, l, Hkv, d]; parts 1 (dQ, writes D to workspace), 2
    (dK/dV, reads D) or 3.  Accumulators are fp32 of the shapes of q and k."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check_cuda(t, n, torch.bfloat16, 4)
    _check_cuda(lse, "lse", torch.float32, 3)
    B, l, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, l, Hkv, d) or v.shape != k.shape or out.shape != q.shape or \
            dout.shape != q.shape or lse.shape != (B, Hq, l):
        raise ValueError("block shapes do not match")
    for t, n, ref in ((dq_acc, "dq_acc", q), (dk_acc, "dk_acc", k), (dv_acc, "dv_acc", k)):
        if t is not None:
            _check_cuda(t, n, torch.float32, 4)
            if t.shape != ref.shape:
                raise ValueError(f"{n} shape does not match")
    if dq is not None:
        _check_cuda(dq, "dq", torch.bfloat16, 4)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    ptr = lambda t: 0 if t is None else t.data_ptr()  # noqa: E731
    with _on(q.device, stream) as sh:
        _lib.ring_attn_bwd_visit(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 dout.data_ptr(), lse.data_ptr(), ptr(dq_acc), ptr(dk_acc),
                                 ptr(dv_acc), ptr(dq), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), B, Hq, Hkv, l, d,
                                 diag, parts, fold_q, fold_kv, scale, sh)


def round_bf16(src: torch.Tensor, dst: torch.Tensor | None = None, stream=None):
    """fp32 -> bf16 (nearest even) through ring_attn_round_bf16."""
    if not src.is_cuda or src.dtype != torch.float32 or not src.is_contiguous():
        raise TypeError("src must be a contiguous fp32 CUDA tensor")
    with _on(src.device, stream) as sh:
        if dst is None:
            dst = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
        _check_out(dst, "dst", torch.bfloat16, tuple(src.shape))
        _lib.ring_attn_round_bf16(src.data_ptr(), dst.data_ptr(), src.numel(), sh)
    return dst


def fwd_visit(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o_acc: torch.Tensor,
              lse_acc: torch.Tensor, diag: int, fold: bool, scale: float | None = None,
              out: torch.Tensor | None = None, stream=None):
    """One ring visit: the query block q [B, l, Hq, d] against the K/V block
    k/v [B, l, Hkv, d] (bf16), written to (fold=False) or folded into
    (fold=True) the running fp32 accumulator o_acc [B, l, Hq, d] and
    lse_acc [B, Hq, l].  ``diag``: 0 every key, 1 keys c <= r, 2 keys c < r
    (local rows).  ``out`` (bf16, optional) receives the rounded
    accumulator.  Returns (o_acc, lse_acc, out)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check_cuda(t, n, torch.bfloat16, 4)
    B, l, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, l, Hkv, d) or v.shape != k.shape:
        raise ValueError(f"k/v shape {tuple(k.shape)}/{tuple(v.shape)} does not match q {tuple(q.shape)}")
    _check_cuda(o_acc, "o_acc", torch.float32, 4)
    _check_cuda(lse_acc, "lse_acc", torch.float32, 3)
    if o_acc.shape != q.shape or lse_acc.shape != (B, Hq, l):
        raise ValueError("o_acc/lse_acc shapes do not match q")
    if out is not None:
        _check_cuda(out, "out", torch.bfloat16, 4)
        if out.shape != q.shape:
            raise ValueError("out shape does not match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on(q.device, stream) as sh:
        _lib.ring_attn_fwd_visit(q.data_ptr(), k.data_ptr(), v.data_ptr(), o_acc.data_ptr(),
                                 lse_acc.data_ptr(), 0 if out is None else out.data_ptr(),
                                 B, Hq, Hkv, l, d, diag, fold, scale, sh)
    return o_acc, lse_acc, out


def quantize_fp8(x: torch.Tensor, codes: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None, stream=None):
    """Block quantisation of x bf16 [B, L, H, d] to E4M3: returns (codes
    uint8 [B, L, H, d], scales fp32 [B, H, ceil(L / 128)]), one scale per
    128-row tile of each (batch, head).  The codes are raw E4M3 bit patterns
    (``codes.view(torch.float8_e4m3fn)`` reads them as FP8)."""
    _check_cuda(x, "x", torch.bfloat16, 4)
    B, L, H, d = x.shape
    with _on(x.device, stream) as sh:
        if codes is None:
            codes = torch.empty((B, L, H, d), dtype=torch.uint8, device=x.device)
        if scales is None:
            scales = torch.empty((B, H, (L + 127) // 128), dtype=torch.float32, device=x.device)
        _check_out(codes, "codes", torch.uint8, (B, L, H, d))
        _check_out(scales, "scales", torch.float32, (B, H, (L + 127) // 128))
        _lib.ring_attn_quantize_fp8(x.data_ptr(), codes.data_ptr(), scales.data_ptr(), B, L, H, d,
                                    sh)
    return codes, scales


def fwd_fp8(q8: torch.Tensor, sq: torch.Tensor, k8: torch.Tensor, sk: torch.Tensor,
            v8: torch.Tensor, sv: torch.Tensor, n_ring: int, causal: bool,
            scale: float | None = None, out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None, stream=None):
    """Ring-ordered attention forward on FP8 inputs from ``quantize_fp8``:
    q8 [B, L, Hq, 128] with sq [B, Hq, L/128], k8/v8 [B, L, Hkv, 128] with
    sk/sv [B, Hkv, L/128].  Returns (out bf16 [B, L, Hq, 128], lse fp32
    [B, Hq, L]).  ``scale`` defaults to 1/sqrt(d)."""
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        _check_cuda(t, n, torch.uint8, 4)
    for t, n in ((sq, "sq"), (sk, "sk"), (sv, "sv")):
        _check_cuda(t, n, torch.float32, 3)
    B, L, Hq, d = q8.shape
    Hkv = k8.shape[2]
    if k8.shape != (B, L, Hkv, d) or v8.shape != k8.shape:
        raise ValueError(f"k8/v8 shape {tuple(k8.shape)}/{tuple(v8.shape)} does not match "
                         f"q8 {tuple(q8.shape)}")
    if L % 128 != 0 or (n_ring > 0 and (L // n_ring) % 128 != 0):
        raise ValueError(f"the FP8 forward needs L / n_ring to be a multiple of 128 "
                         f"(L={L}, n_ring={n_ring})")
    T = L // 128
    if sq.shape != (B, Hq, T) or sk.shape != (B, Hkv, T) or sv.shape != (B, Hkv, T):
        raise ValueError("scale tensors must be [B, H, L/128]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with _on(q8.device, stream) as sh:
        if out is None:
            out = torch.empty((B, L, Hq, d), dtype=torch.bfloat16, device=q8.device)
        if lse is None:
            lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q8.device)
        _check_out(out, "out", torch.bfloat16, (B, L, Hq, d))
        _check_out(lse, "lse", torch.float32, (B, Hq, L))
        _lib.ring_attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), sq.data_ptr(),
                               sk.data_ptr(), sv.data_ptr(), out.data_ptr(), lse.data_ptr(), B,
                               Hq, Hkv, L, d, n_ring, causal, scale, sh)
    return out, lse


def merge(o_a: torch.Tensor, lse_a: torch.Tensor, o_b: torch.Tensor, lse_b: torch.Tensor,
          out: torch.Tensor | None = None, lse_out: torch.Tensor | None = None, stream=None):
    """Log-sum-exp merge of two partials: o [rows, d] fp32, lse [rows] fp32."""
    _check_cuda(o_a, "o_a", torch.float32, 2)
    _check_cuda(o_b, "o_b", torch.float32, 2)
    _check_cuda(lse_a, "lse_a", torch.float32, 1)
    _check_cuda(lse_b, "lse_b", torch.float32, 1)
    rows, d = o_a.shape
    if tuple(o_b.shape) != (rows, d) or tuple(lse_a.shape) != (rows,) or tuple(lse_b.shape) != (rows,):
        raise ValueError("o_a, o_b must be [rows, d] and lse_a, lse_b [rows]")
    with _on(o_a.device, stream) as sh:
        if out is None:
            out = torch.empty_like(o_a)
        if lse_out is None:
            lse_out = torch.empty_like(lse_a)
        _check_out(out, "out", torch.float32, (rows, d))
        _check_out(lse_out, "lse_out", torch.float32, (rows,))
        _lib.ring_attn_merge(o_a.data_ptr(), lse_a.data_ptr(), o_b.data_ptr(), lse_b.data_ptr(),
                             out.data_ptr(), lse_out.data_ptr(), rows, d, sh)
    return out, lse_out


def check_status(stream=None):
    with torch.cuda.device(torch.cuda.current_device()):
        _lib.ring_attn_check_status(_stream_handle(stream))


class _RingAttention(torch.autograd.Function):
    """Autograd bridge: forward through ring_attn_fwd (saving out and lse),
    backward through ring_attn_bwd."""

    @staticmethod
    def forward(ctx, q, k, v, n_ring, causal, scale):
        out, lse = fwd(q, k, v, n_ring, causal, scale)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.n_ring, ctx.causal, ctx.scale = n_ring, causal, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, out, lse = ctx.saved_tensors
        dq, dk, dv = bwd(q, k, v, out, dout.contiguous().to(torch.bfloat16), lse, ctx.n_ring,
                         ctx.causal, ctx.scale)
        return dq, dk, dv, None, None, None


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_ring: int, causal: bool,
              scale: float | None = None) -> torch.Tensor:
    """Differentiable ring-ordered attention on one GPU: the output of
    ``fwd``, with gradients for q, k and v from ``bwd``."""
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return _RingAttention.apply(q, k, v, n_ring, causal, scale)
