"""B200-native ring-ordered blockwise attention.

The product is the C-ABI library ``libring_attn.so`` (kernels for sm_100a,
declared in ``include/ring_attn.h``: forward, backward, their per-visit
forms, the log-sum-exp merge, and the FP8 forward with its block quantiser).
This package holds its sources (``csrc/``), the in-tree build (``build``),
the ctypes binding (``_lib``), a torch-facing
wrapper (``api``) that only marshals tensors into the C calls, the
multi-process ring over torch.distributed with its contiguous, zigzag and
striped layouts (``ring``), and the seeded synthetic inputs (``inputs``).
"""

from ._lib import (  # noqa: F401
    RingAttnError,
    ring_attn_bwd,
    ring_attn_bwd_noalloc,
    ring_attn_bwd_visit,
    ring_attn_bwd_workspace_size,
    ring_attn_check_status,
    ring_attn_debug_inject,
    ring_attn_fwd,
    ring_attn_fwd_fp8,
    ring_attn_fwd_visit,
    ring_attn_merge,
    ring_attn_quantize_fp8,
    ring_attn_round_bf16,
    ring_attn_set_max_ctas,
    ring_attn_set_schedule,
    ring_attn_set_wait_limit_ns,
    ring_attn_version,
)
