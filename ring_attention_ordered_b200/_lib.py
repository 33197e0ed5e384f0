"""ctypes binding of libring_attn.so (argument marshalling only).

The functions here have the names and arguments of the C ABI in
``include/ring_attn.h``; they take raw device pointers (ints) and a CUDA
stream handle (int, 0 = legacy default stream).  A non-OK status raises
:class:`RingAttnError`.  There is no fallback: if the shared library is
missing the first call raises.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libring_attn.so")

RA_OK, RA_ERR_INVALID_ARG, RA_ERR_UNSUPPORTED, RA_ERR_CUDA, RA_ERR_TIMEOUT = range(5)

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
SIGNATURES = {
    "ring_attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I, ctypes.c_float, _P]),
    "ring_attn_fwd_visit": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I,
                                 ctypes.c_float, _P]),
    "ring_attn_bwd_workspace_size": (_I, [_I, _I, _I64, ctypes.POINTER(ctypes.c_size_t)]),
    "ring_attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I64,
                           _I, _I, _I, ctypes.c_float, _P]),
    "ring_attn_bwd_visit": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I,
                                 _I, _I64, _I, _I, _I, _I, _I, ctypes.c_float, _P]),
    "ring_attn_round_bf16": (_I, [_P, _P, _I64, _P]),
    "ring_attn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I,
                                   ctypes.c_float, _P]),
    "ring_attn_quantize_fp8": (_I, [_P, _P, _P, _I, _I64, _I, _I, _P]),
    "ring_attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I64, _I, _I, _I,
                               ctypes.c_float, _P]),
    "ring_attn_merge": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I, _P]),
    "ring_attn_check_status": (_I, [_P]),
    "ring_attn_set_wait_limit_ns": (_I, [ctypes.c_uint64]),
    "ring_attn_set_max_ctas": (_I, [_I]),
    "ring_attn_set_schedule": (_I, [_I]),
    "ring_attn_debug_inject": (_I, [ctypes.c_uint]),
    "ring_attn_status_string": (ctypes.c_char_p, [_I]),
    "ring_attn_last_error": (ctypes.c_char_p, []),
    "ring_attn_version": (_I, []),
}


class RingAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{status_string(status)}: {message}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library once; raises OSError if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} is missing; build it with "
                          "`python -m ring_attention_ordered_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().ring_attn_status_string(status).decode()


def last_error() -> str:
    return load().ring_attn_last_error().decode()


def _check(status: int) -> int:
    if status != RA_OK:
        raise RingAttnError(status, last_error())
    return status


def ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, L, d, n_ring, causal, scale, stream=0):
    return _check(load().ring_attn_fwd(q, k, v, out, lse, B, Hq, Hkv, L, d, n_ring,
                                       int(bool(causal)), float(scale), stream))


def ring_attn_bwd_workspace_size(B, Hq, L):
    n = ctypes.c_size_t(0)
    _check(load().ring_attn_bwd_workspace_size(B, Hq, L, ctypes.byref(n)))
    return n.value


def ring_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, L,
                  d, n_ring, causal, scale, stream=0):
    return _check(load().ring_attn_bwd(q, k, v, out, dout, lse, dq, dk, dv, workspace,
                                       workspace_bytes, B, Hq, Hkv, L, d, n_ring,
                                       int(bool(causal)), float(scale), stream))


def ring_attn_bwd_visit(q, k, v, out, dout, lse, dq_acc, dk_acc, dv_acc, dq, workspace,
                        workspace_bytes, B, Hq, Hkv, l, d, diag, parts, fold_q, fold_kv, scale,
                        stream=0):
    return _check(load().ring_attn_bwd_visit(q, k, v, out, dout, lse, dq_acc, dk_acc, dv_acc, dq,
                                             workspace, workspace_bytes, B, Hq, Hkv, l, d,
                                             int(diag), int(parts), int(fold_q), int(fold_kv),
                                             float(scale), stream))


def ring_attn_round_bf16(src, dst, n, stream=0):
    return _check(load().ring_attn_round_bf16(src, dst, n, stream))


def ring_attn_bwd_noalloc(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv, L, d, n_ring, causal,
                          scale, stream=0):
    return _check(load().ring_attn_bwd_noalloc(q, k, v, out, dout, lse, dq, dk, dv, B, Hq, Hkv,
                                               L, d, n_ring, int(bool(causal)), float(scale),
                                               stream))


def ring_attn_fwd_visit(q, k, v, o_acc, lse_acc, out, B, Hq, Hkv, l, d, diag, fold, scale,
                        stream=0):
    return _check(load().ring_attn_fwd_visit(q, k, v, o_acc, lse_acc, out, B, Hq, Hkv, l, d,
                                             int(diag), int(fold), float(scale), stream))


def ring_attn_quantize_fp8(x, codes, scales, B, L, H, d, stream=0):
    return _check(load().ring_attn_quantize_fp8(x, codes, scales, B, L, H, d, stream))


def ring_attn_fwd_fp8(q8, k8, v8, sq, sk, sv, out, lse, B, Hq, Hkv, L, d, n_ring, causal, scale,
                      stream=0):
    return _check(load().ring_attn_fwd_fp8(q8, k8, v8, sq, sk, sv, out, lse, B, Hq, Hkv, L, d,
                                           n_ring, int(bool(causal)), float(scale), stream))


def ring_attn_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d, stream=0):
    return _check(load().ring_attn_merge(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, d, stream))


def ring_attn_check_status(stream=0):
    return _check(load().ring_attn_check_status(stream))


def ring_attn_set_wait_limit_ns(ns: int):
    return _check(load().ring_attn_set_wait_limit_ns(ns))


def ring_attn_set_max_ctas(n: int):
    return _check(load().ring_attn_set_max_ctas(n))


RA_SCHEDULE_AUTO, RA_SCHEDULE_LONGEST_FIRST, RA_SCHEDULE_HEAD_MAJOR = 0, 1, 2


def ring_attn_set_schedule(schedule: int):
    return _check(load().ring_attn_set_schedule(schedule))


def ring_attn_debug_inject(flags: int):
    return _check(load().ring_attn_debug_inject(flags))


def ring_attn_version() -> int:
    return load().ring_attn_version()
