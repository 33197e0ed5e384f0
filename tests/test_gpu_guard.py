"""Out-of-bounds writes, caught without a sanitizer: every output buffer of a
call sits inside a larger allocation whose bands on both sides hold a byte
pattern; after the call the bands must be unchanged and the result must be
bitwise the one written to a plain buffer.  Shapes have ragged tiles (blocks
that are not a multiple of 128 rows) and ragged quantisation tiles, where an
unmasked store would land past the end.  Also: the torch wrapper refuses
outputs of the wrong shape (the library writes through raw pointers and
cannot see a buffer's size)."""

from __future__ import annotations

import math

import pytest
import torch

pytestmark = pytest.mark.gpu

PAD = 1 << 16
PATTERN = 0xA5


@pytest.fixture(scope="module")
def ra():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import _lib, api
    _lib.load()
    return api


class Guarded:
    """A tensor of ``shape`` and ``dtype`` at byte offset PAD of a buffer
    whose first and last PAD bytes hold PATTERN."""

    def __init__(self, shape, dtype, fill=None):
        esize = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape) * esize
        self.buf = torch.full((self.n + 2 * PAD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.buf[PAD:PAD + self.n].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def bands_intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.buf[:PAD] == PATTERN).all()) and bool((self.buf[PAD + self.n:] == PATTERN).all())


def _inputs(B, Hq, Hkv, L, d, seed):
    from ring_attention_ordered_b200.inputs import make_inputs
    return (t.cuda() for t in make_inputs(B, Hq, Hkv, L, d, seed=seed))


@pytest.mark.parametrize("B,Hq,Hkv,L,d,n_ring,causal", [
    (1, 4, 1, 600, 128, 3, True),     # blocks of 200 rows
    (2, 2, 2, 200, 64, 5, False),     # blocks of 40 rows
    (1, 2, 2, 512, 128, 4, True),
])
def test_forward_and_backward_stay_in_bounds(ra, B, Hq, Hkv, L, d, n_ring, causal):
    from ring_attention_ordered_b200 import _lib
    q, k, v = _inputs(B, Hq, Hkv, L, d, seed=900 + L + d)
    out, lse = Guarded((B, L, Hq, d), torch.bfloat16), Guarded((B, Hq, L), torch.float32)
    ra.fwd(q, k, v, n_ring, causal, out=out.t, lse=lse.t)
    ra.check_status()
    assert out.bands_intact() and lse.bands_intact()
    o_ref, l_ref = ra.fwd(q, k, v, n_ring, causal)
    ra.check_status()
    assert torch.equal(out.t, o_ref) and torch.equal(lse.t, l_ref)

    g = torch.Generator().manual_seed(L)
    do = torch.randn((B, L, Hq, d), generator=g).to(torch.bfloat16).cuda()
    dq, dk, dv = (Guarded(tuple(t.shape), torch.bfloat16) for t in (q, k, v))
    ws = Guarded((_lib.ring_attn_bwd_workspace_size(B, Hq, L),), torch.uint8)
    ra.bwd(q, k, v, o_ref, do, l_ref, n_ring, causal, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    ra.check_status()
    assert all(x.bands_intact() for x in (dq, dk, dv, ws))
    g_ref = ra.bwd(q, k, v, o_ref, do, l_ref, n_ring, causal)
    ra.check_status()
    assert all(torch.equal(x.t, y) for x, y in zip((dq, dk, dv), g_ref))


def test_visit_and_merge_stay_in_bounds(ra):
    q, k, v = _inputs(1, 4, 2, 200, 128, seed=31)
    o_acc = Guarded((1, 200, 4, 128), torch.float32)
    lse_acc = Guarded((1, 4, 200), torch.float32)
    out = Guarded((1, 200, 4, 128), torch.bfloat16)
    ra.fwd_visit(q, k, v, o_acc.t, lse_acc.t, 1, False, out=out.t)
    ra.fwd_visit(q, k.flip(1).contiguous(), v, o_acc.t, lse_acc.t, 0, True, out=out.t)
    ra.check_status()
    assert o_acc.bands_intact() and lse_acc.bands_intact() and out.bands_intact()

    rows = 1000
    g = torch.Generator().manual_seed(5)
    o_a, o_b = (torch.randn(rows, 64, generator=g).cuda() for _ in range(2))
    l_a, l_b = (torch.randn(rows, generator=g).cuda() for _ in range(2))
    mo, ml = Guarded((rows, 64), torch.float32), Guarded((rows,), torch.float32)
    ra.merge(o_a, l_a, o_b, l_b, out=mo.t, lse_out=ml.t)
    assert mo.bands_intact() and ml.bands_intact()
    r_o, r_l = ra.merge(o_a, l_a, o_b, l_b)
    torch.cuda.synchronize()
    assert torch.equal(mo.t, r_o) and torch.equal(ml.t, r_l)

    src = torch.randn(1000, 8, generator=g).cuda()
    dst = Guarded((1000, 8), torch.bfloat16)
    ra.round_bf16(src, dst.t)
    assert dst.bands_intact() and torch.equal(dst.t, src.to(torch.bfloat16))


def test_fp8_paths_stay_in_bounds(ra):
    x = next(_inputs(1, 2, 2, 300, 64, seed=41))
    codes = Guarded((1, 300, 2, 64), torch.uint8)
    scales = Guarded((1, 2, 3), torch.float32)
    ra.quantize_fp8(x, codes.t, scales.t)
    ra.check_status()
    assert codes.bands_intact() and scales.bands_intact()
    c_ref, s_ref = ra.quantize_fp8(x)
    torch.cuda.synchronize()
    assert torch.equal(codes.t, c_ref) and torch.equal(scales.t, s_ref)

    q, k, v = _inputs(1, 3, 1, 512, 128, seed=42)
    q8, sq = ra.quantize_fp8(q)
    k8, sk = ra.quantize_fp8(k)
    v8, sv = ra.quantize_fp8(v)
    out, lse = Guarded((1, 512, 3, 128), torch.bfloat16), Guarded((1, 3, 512), torch.float32)
    ra.fwd_fp8(q8, sq, k8, sk, v8, sv, 2, True, out=out.t, lse=lse.t)
    ra.check_status()
    assert out.bands_intact() and lse.bands_intact()
    o_ref, l_ref = ra.fwd_fp8(q8, sq, k8, sk, v8, sv, 2, True)
    ra.check_status()
    assert torch.equal(out.t, o_ref) and torch.equal(lse.t, l_ref)


def test_wrapper_refuses_wrong_output_shapes(ra):
    q, k, v = _inputs(1, 2, 2, 256, 64, seed=51)
    with pytest.raises(ValueError):
        ra.fwd(q, k, v, 2, True, out=torch.empty((1, 128, 2, 64), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        ra.fwd(q, k, v, 2, True, lse=torch.empty((1, 2, 128), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        ra.round_bf16(torch.zeros(64, device="cuda"), torch.empty(32, dtype=torch.bfloat16, device="cuda"))
    o = torch.zeros(16, 64, device="cuda")
    l_ = torch.zeros(16, device="cuda")
    with pytest.raises(ValueError):
        ra.merge(o, l_, o, l_, out=torch.empty(8, 64, device="cuda"))
    with pytest.raises(ValueError):
        ra.quantize_fp8(q, torch.empty((1, 256, 2, 32), dtype=torch.uint8, device="cuda"))
