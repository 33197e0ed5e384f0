"""ring_attn_bwd_noalloc: the backward pass with its D vector in the
library's fixed device array instead of a caller workspace.

Collected last on purpose (file name), so that the GPU test also runs after
every other test of the session has used the library on the same device."""

from __future__ import annotations

import pytest
import torch

from ring_attention_ordered_b200 import _lib


def test_oversize_is_rejected_before_any_launch():
    """B*Hq*L above the fixed array's 1,048,576 rows: a clear argument error,
    checked on the host before any device work (fake, never-used pointers)."""
    p = 1 << 20
    with pytest.raises(_lib.RingAttnError) as ei:
        _lib.ring_attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 32, 32, 1 << 16, 128, 8, 1,
                                   0.088, 0)
    assert ei.value.status == _lib.RA_ERR_INVALID_ARG
    assert "static scratch" in _lib.last_error()


def test_empty_problem_needs_no_device():
    assert _lib.ring_attn_bwd_noalloc(0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 4, 2, 256, 128, 2, 1, 0.1,
                                      0) == _lib.RA_OK


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    """Two different problems back to back through ring_attn_bwd_noalloc give
    bitwise the gradients of ring_attn_bwd with a workspace (the second call
    reuses the fixed array the first one filled)."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ring_attention_ordered_b200 import api
    from ring_attention_ordered_b200.inputs import make_grad_output, make_inputs
    for (B, Hq, Hkv, L, d, n_ring, causal, seed) in ((1, 4, 2, 1024, 128, 4, True, 41),
                                                      (2, 2, 2, 600, 64, 3, False, 42)):
        q, k, v = (t.cuda() for t in make_inputs(B, Hq, Hkv, L, d, seed=seed))
        do = make_grad_output(B, L, Hq, d, seed).cuda()
        out, lse = api.fwd(q, k, v, n_ring, causal)
        ref = api.bwd(q, k, v, out, do, lse, n_ring, causal)
        got = api.bwd_noalloc(q, k, v, out, do, lse, torch.empty_like(q), torch.empty_like(k),
                              torch.empty_like(v), n_ring, causal)
        api.check_status()
        for a, b in zip(got, ref):
            assert torch.equal(a, b), (B, Hq, L)
