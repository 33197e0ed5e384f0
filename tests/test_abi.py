"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects invalid arguments before touching the device."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

from ring_attention_ordered_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ring_attn.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from ring_attention_ordered_b200 import build
        build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ring_attn_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    assert "ring_attn_fwd" in names and "ring_attn_merge" in names
    assert set(names) == set(_lib.SIGNATURES), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version(lib):
    for code, name in enumerate(["RA_OK", "RA_ERR_INVALID_ARG", "RA_ERR_UNSUPPORTED",
                                 "RA_ERR_CUDA", "RA_ERR_TIMEOUT"]):
        assert _lib.status_string(code) == name
    assert _lib.status_string(99) == "RA_ERR_UNKNOWN"
    assert _lib.ring_attn_version() == 104


# Fake, never-dereferenced device addresses: validation rejects these calls
# before any CUDA call is made.
A = 1 << 20
Q, K, V, O, LSE = A, 2 * A * 64, 3 * A * 64, 4 * A * 64, 5 * A * 64


def fwd_status(lib, **kw):
    args = dict(q=Q, k=K, v=V, out=O, lse=LSE, B=1, Hq=2, Hkv=2, L=512, d=128, n_ring=4,
                causal=1, scale=0.088)
    args.update(kw)
    return lib.ring_attn_fwd(args["q"], args["k"], args["v"], args["out"], args["lse"],
                             args["B"], args["Hq"], args["Hkv"], args["L"], args["d"],
                             args["n_ring"], args["causal"], args["scale"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(L=510), _lib.RA_ERR_INVALID_ARG),            # blocks would be unequal
    (dict(n_ring=0), _lib.RA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), _lib.RA_ERR_INVALID_ARG),
    (dict(Hkv=0), _lib.RA_ERR_INVALID_ARG),
    (dict(B=-1), _lib.RA_ERR_INVALID_ARG),
    (dict(causal=2), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=-0.5), _lib.RA_ERR_INVALID_ARG),
    (dict(d=96), _lib.RA_ERR_UNSUPPORTED),
    (dict(d=256), _lib.RA_ERR_UNSUPPORTED),
    (dict(q=0), _lib.RA_ERR_INVALID_ARG),
    (dict(lse=0), _lib.RA_ERR_INVALID_ARG),
    (dict(k=K + 8), _lib.RA_ERR_INVALID_ARG),           # not 16-byte aligned
    (dict(out=Q + 64), _lib.RA_ERR_INVALID_ARG),        # output overlaps q
    (dict(lse=O + 16), _lib.RA_ERR_INVALID_ARG),        # lse overlaps out
    (dict(B=1, L=1 << 31, n_ring=1), _lib.RA_ERR_INVALID_ARG),
])
def test_fwd_rejects_invalid_arguments(lib, kw, status):
    assert fwd_status(lib, **kw) == status
    assert _lib.last_error()


@pytest.mark.parametrize("kw", [dict(B=0), dict(L=0), dict(Hq=0, Hkv=0)])
def test_fwd_empty_problem_launches_nothing(lib, kw):
    assert fwd_status(lib, q=0, k=0, v=0, out=0, lse=0, **kw) == _lib.RA_OK


OACC = 6 * A * 64


def visit_status(lib, **kw):
    args = dict(q=Q, k=K, v=V, o_acc=OACC, lse_acc=LSE, out=O, B=1, Hq=2, Hkv=2, l=512, d=128,
                diag=1, fold=1, scale=0.088)
    args.update(kw)
    return lib.ring_attn_fwd_visit(args["q"], args["k"], args["v"], args["o_acc"],
                                   args["lse_acc"], args["out"], args["B"], args["Hq"],
                                   args["Hkv"], args["l"], args["d"], args["diag"], args["fold"],
                                   args["scale"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(diag=3), _lib.RA_ERR_INVALID_ARG),
    (dict(diag=-1), _lib.RA_ERR_INVALID_ARG),
    (dict(fold=2), _lib.RA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.RA_ERR_INVALID_ARG),
    (dict(d=96), _lib.RA_ERR_UNSUPPORTED),
    (dict(o_acc=0), _lib.RA_ERR_INVALID_ARG),
    (dict(lse_acc=0), _lib.RA_ERR_INVALID_ARG),
    (dict(o_acc=OACC + 4), _lib.RA_ERR_INVALID_ARG),     # not 16-byte aligned
    (dict(out=O + 8), _lib.RA_ERR_INVALID_ARG),
    (dict(o_acc=Q + 64), _lib.RA_ERR_INVALID_ARG),      # accumulator overlaps q
    (dict(out=OACC + 4096), _lib.RA_ERR_INVALID_ARG),   # out overlaps the accumulator
    (dict(lse_acc=OACC + 16), _lib.RA_ERR_INVALID_ARG),
    (dict(B=1, l=1 << 31), _lib.RA_ERR_INVALID_ARG),
])
def test_visit_rejects_invalid_arguments(lib, kw, status):
    assert visit_status(lib, **kw) == status
    assert _lib.last_error()


@pytest.mark.parametrize("kw", [dict(B=0), dict(l=0), dict(Hq=0, Hkv=0)])
def test_visit_empty_problem_launches_nothing(lib, kw):
    assert visit_status(lib, q=0, k=0, v=0, o_acc=0, lse_acc=0, out=0, **kw) == _lib.RA_OK


def merge_status(lib, rows=64, d=128, **kw):
    p = dict(o_a=A, lse_a=2 * A, o_b=3 * A, lse_b=4 * A, o_out=5 * A, lse_out=6 * A)
    p.update(kw)
    return lib.ring_attn_merge(p["o_a"], p["lse_a"], p["o_b"], p["lse_b"], p["o_out"],
                               p["lse_out"], rows, d, None)


@pytest.mark.parametrize("kw,status", [
    (dict(rows=-1), _lib.RA_ERR_INVALID_ARG),
    (dict(d=6), _lib.RA_ERR_INVALID_ARG),
    (dict(d=0), _lib.RA_ERR_INVALID_ARG),
    (dict(o_a=0), _lib.RA_ERR_INVALID_ARG),
    (dict(lse_b=4 * A + 4), _lib.RA_ERR_INVALID_ARG),
    (dict(o_out=A + 16), _lib.RA_ERR_INVALID_ARG),     # partial overlap with o_a
    (dict(lse_out=5 * A), _lib.RA_ERR_INVALID_ARG),    # lse_out inside o_out
])
def test_merge_rejects_invalid_arguments(lib, kw, status):
    assert merge_status(lib, **kw) == status


def test_merge_zero_rows_is_ok(lib):
    assert merge_status(lib, rows=0, o_a=0, lse_a=0, o_b=0, lse_b=0, o_out=0, lse_out=0) == _lib.RA_OK


def test_options_validate(lib):
    assert lib.ring_attn_set_max_ctas(-1) == _lib.RA_ERR_INVALID_ARG
    assert lib.ring_attn_set_max_ctas(0) == _lib.RA_OK
    assert lib.ring_attn_debug_inject(2) == _lib.RA_ERR_INVALID_ARG
    assert lib.ring_attn_debug_inject(0) == _lib.RA_OK
    assert lib.ring_attn_set_wait_limit_ns(0) == _lib.RA_OK
    assert lib.ring_attn_set_schedule(3) == _lib.RA_ERR_INVALID_ARG
    for sched in (_lib.RA_SCHEDULE_LONGEST_FIRST, _lib.RA_SCHEDULE_HEAD_MAJOR, _lib.RA_SCHEDULE_AUTO):
        assert lib.ring_attn_set_schedule(sched) == _lib.RA_OK


def test_python_binding_raises_on_error(lib):
    with pytest.raises(_lib.RingAttnError) as ei:
        _lib.ring_attn_fwd(Q, K, V, O, LSE, 1, 2, 2, 510, 128, 4, 1, 0.1, 0)
    assert ei.value.status == _lib.RA_ERR_INVALID_ARG
    assert "equal blocks" in str(ei.value)


DO, DQ, DK, DV, WS = (7 * A * 64, 8 * A * 64, 9 * A * 64, 10 * A * 64, 11 * A * 64)


def bwd_status(lib, **kw):
    args = dict(q=Q, k=K, v=V, out=O, dout=DO, lse=LSE, dq=DQ, dk=DK, dv=DV, ws=WS,
                ws_bytes=1 << 20, B=1, Hq=2, Hkv=2, L=512, d=128, n_ring=4, causal=1, scale=0.088)
    args.update(kw)
    return lib.ring_attn_bwd(args["q"], args["k"], args["v"], args["out"], args["dout"],
                             args["lse"], args["dq"], args["dk"], args["dv"], args["ws"],
                             args["ws_bytes"], args["B"], args["Hq"], args["Hkv"], args["L"],
                             args["d"], args["n_ring"], args["causal"], args["scale"], None)


def test_bwd_workspace_size():
    assert _lib.ring_attn_bwd_workspace_size(2, 8, 8192) == 2 * 8 * 8192 * 4
    assert _lib.ring_attn_bwd_workspace_size(0, 8, 8192) == 0
    with pytest.raises(_lib.RingAttnError):
        _lib.ring_attn_bwd_workspace_size(-1, 8, 8192)


@pytest.mark.parametrize("kw,status", [
    (dict(L=510), _lib.RA_ERR_INVALID_ARG),
    (dict(n_ring=0), _lib.RA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), _lib.RA_ERR_INVALID_ARG),
    (dict(causal=2), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), _lib.RA_ERR_INVALID_ARG),
    (dict(d=96), _lib.RA_ERR_UNSUPPORTED),
    (dict(dout=0), _lib.RA_ERR_INVALID_ARG),
    (dict(ws=0), _lib.RA_ERR_INVALID_ARG),
    (dict(ws_bytes=1 * 2 * 512 * 4 - 4), _lib.RA_ERR_INVALID_ARG),   # workspace too small
    (dict(dq=DQ + 8), _lib.RA_ERR_INVALID_ARG),                       # not 16-byte aligned
    (dict(dk=Q + 64), _lib.RA_ERR_INVALID_ARG),                       # dk overlaps q
    (dict(ws=DV + 64), _lib.RA_ERR_INVALID_ARG),                      # workspace overlaps dv
    (dict(dv=LSE), _lib.RA_ERR_INVALID_ARG),                          # dv overlaps lse
])
def test_bwd_rejects_invalid_arguments(lib, kw, status):
    assert bwd_status(lib, **kw) == status
    assert _lib.last_error()


@pytest.mark.parametrize("kw", [dict(B=0), dict(L=0), dict(Hq=0, Hkv=0)])
def test_bwd_empty_problem_launches_nothing(lib, kw):
    assert bwd_status(lib, q=0, k=0, v=0, out=0, dout=0, lse=0, dq=0, dk=0, dv=0, ws=0,
                      ws_bytes=0, **kw) == _lib.RA_OK


def bwd_visit_status(lib, **kw):
    args = dict(q=Q, k=K, v=V, out=O, dout=DO, lse=LSE, dq_acc=DQ, dk_acc=DK, dv_acc=DV, dq=0,
                ws=WS, ws_bytes=1 << 20, B=1, Hq=2, Hkv=2, l=512, d=128, diag=1, parts=3,
                fold_q=1, fold_kv=1, scale=0.088)
    args.update(kw)
    a = args
    return lib.ring_attn_bwd_visit(a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"],
                                   a["dq_acc"], a["dk_acc"], a["dv_acc"], a["dq"], a["ws"],
                                   a["ws_bytes"], a["B"], a["Hq"], a["Hkv"], a["l"], a["d"],
                                   a["diag"], a["parts"], a["fold_q"], a["fold_kv"], a["scale"],
                                   None)


@pytest.mark.parametrize("kw,status", [
    (dict(diag=3), _lib.RA_ERR_INVALID_ARG),
    (dict(parts=0), _lib.RA_ERR_INVALID_ARG),
    (dict(parts=4), _lib.RA_ERR_INVALID_ARG),
    (dict(fold_q=2), _lib.RA_ERR_INVALID_ARG),
    (dict(d=96), _lib.RA_ERR_UNSUPPORTED),
    (dict(parts=1, dq_acc=0), _lib.RA_ERR_INVALID_ARG),
    (dict(parts=2, dk_acc=0), _lib.RA_ERR_INVALID_ARG),
    (dict(ws_bytes=100), _lib.RA_ERR_INVALID_ARG),
    (dict(dq_acc=DQ + 4), _lib.RA_ERR_INVALID_ARG),
    (dict(dk_acc=K + 64), _lib.RA_ERR_INVALID_ARG),      # accumulator overlaps k
    (dict(dv_acc=DK + 64), _lib.RA_ERR_INVALID_ARG),     # accumulators overlap
])
def test_bwd_visit_rejects_invalid_arguments(lib, kw, status):
    assert bwd_visit_status(lib, **kw) == status
    assert _lib.last_error()


def test_round_bf16_validation(lib):
    assert lib.ring_attn_round_bf16(DQ, DK, 0, None) == _lib.RA_OK
    assert lib.ring_attn_round_bf16(DQ, DK, 12, None) == _lib.RA_ERR_INVALID_ARG      # n % 8
    assert lib.ring_attn_round_bf16(DQ + 4, DK, 16, None) == _lib.RA_ERR_INVALID_ARG  # alignment
    assert lib.ring_attn_round_bf16(DQ, DQ + 16, 16, None) == _lib.RA_ERR_INVALID_ARG  # overlap


SQ, SK, SV = 7 * A * 64, 8 * A * 64, 9 * A * 64


def fp8_status(lib, **kw):
    args = dict(q8=Q, k8=K, v8=V, sq=SQ, sk=SK, sv=SV, out=O, lse=LSE, B=1, Hq=2, Hkv=2, L=512,
                d=128, n_ring=4, causal=1, scale=0.088)
    args.update(kw)
    return lib.ring_attn_fwd_fp8(args["q8"], args["k8"], args["v8"], args["sq"], args["sk"],
                                 args["sv"], args["out"], args["lse"], args["B"], args["Hq"],
                                 args["Hkv"], args["L"], args["d"], args["n_ring"],
                                 args["causal"], args["scale"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=64), _lib.RA_ERR_UNSUPPORTED),              # FP8 forward is d = 128 only
    (dict(n_ring=8), _lib.RA_ERR_UNSUPPORTED),          # blocks of 64 rows
    (dict(L=510), _lib.RA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), _lib.RA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.RA_ERR_INVALID_ARG),
    (dict(causal=3), _lib.RA_ERR_INVALID_ARG),
    (dict(sq=0), _lib.RA_ERR_INVALID_ARG),
    (dict(sk=SK + 4), _lib.RA_ERR_INVALID_ARG),         # not 16-byte aligned
    (dict(out=Q + 4096), _lib.RA_ERR_INVALID_ARG),      # output overlaps q8
    (dict(lse=SV), _lib.RA_ERR_INVALID_ARG),            # lse overlaps sv
    (dict(lse=O + 64), _lib.RA_ERR_INVALID_ARG),        # lse overlaps out
])
def test_fwd_fp8_rejects_invalid_arguments(lib, kw, status):
    assert fp8_status(lib, **kw) == status
    assert _lib.last_error()


@pytest.mark.parametrize("kw", [dict(B=0), dict(L=0), dict(Hq=0, Hkv=0)])
def test_fwd_fp8_empty_problem_launches_nothing(lib, kw):
    assert fp8_status(lib, q8=0, k8=0, v8=0, sq=0, sk=0, sv=0, out=0, lse=0, **kw) == _lib.RA_OK


def quant_status(lib, **kw):
    args = dict(x=Q, codes=K, scales=SQ, B=1, L=300, H=2, d=128)
    args.update(kw)
    return lib.ring_attn_quantize_fp8(args["x"], args["codes"], args["scales"], args["B"],
                                      args["L"], args["H"], args["d"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=12), _lib.RA_ERR_UNSUPPORTED),
    (dict(d=0), _lib.RA_ERR_UNSUPPORTED),
    (dict(d=264), _lib.RA_ERR_UNSUPPORTED),
    (dict(H=70000), _lib.RA_ERR_UNSUPPORTED),
    (dict(B=-1), _lib.RA_ERR_INVALID_ARG),
    (dict(x=0), _lib.RA_ERR_INVALID_ARG),
    (dict(codes=K + 8), _lib.RA_ERR_INVALID_ARG),       # not 16-byte aligned
    (dict(scales=SQ + 2), _lib.RA_ERR_INVALID_ARG),     # not 4-byte aligned
    (dict(codes=Q + 64), _lib.RA_ERR_INVALID_ARG),      # codes overlap x
    (dict(scales=K + 16), _lib.RA_ERR_INVALID_ARG),     # scales overlap codes
])
def test_quantize_fp8_rejects_invalid_arguments(lib, kw, status):
    assert quant_status(lib, **kw) == status
    assert _lib.last_error()


@pytest.mark.parametrize("kw", [dict(B=0), dict(L=0), dict(H=0)])
def test_quantize_fp8_empty_launches_nothing(lib, kw):
    assert quant_status(lib, x=0, codes=0, scales=0, **kw) == _lib.RA_OK
