"""fp64 CPU oracle for ring-ordered blockwise attention.

This package is TEST INFRASTRUCTURE. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
The product path (the CUDA library and its Python binding) never calls it and
shares no code with it: the two meet only through the seeded inputs.

Every function cites the passage of the source pages it restates; the pages
are

* "Ring Attention 环注意力" (slowleelab, ai-terms-fun) -- the primary page,
  cited by its layer and section (L3 definition, L4 §4.2 algorithm, §4.3
  fusion with FlashAttention, §4.5 limitations, L5 §5.2 pitfalls);
* the FlashAttention / PagedAttention article (developer.aliyun), section 二
  (FlashAttention core principle, FlashAttention-2, FlashAttention-3);
* "大模型底层原理注意力机制优化与长上下文处理" (lnwmold), §2.1 (standard
  self-attention) and §2.2 (MQA/GQA).

``attn_fp64`` holds the forward pass and the ring; ``attn_bwd_fp64`` the
gradients of the same definition (the backward pass the FlashAttention
article's recomputation serves); ``fp8_fp64`` the E4M3 format, the block
quantisation of the FP8 forward (FlashAttention article, FlashAttention-3)
and the attention of the dequantised tensors.

Every function here has a pin in ``tests/test_oracle.py``,
``tests/test_oracle_bwd.py`` or ``tests/test_oracle_fp8.py`` against something
other than itself (a library routine, a closed form, an invariant, the pages'
worked example, or brute force on tiny inputs); none is parity unpinned.
"""

from .attn_fp64 import (  # noqa: F401
    NEG_INF,
    attention,
    attention_rows,
    attention_probs,
    block_attention,
    brute_attention,
    ring_order,
    ring_visits,
    ring_attention,
    ring_attention_merged,
    merge,
    causal_pair_counts,
    kv_bytes_per_ring_step,
)
from .attn_bwd_fp64 import (  # noqa: F401
    attention_bwd,
    attention_bwd_dq_rows,
    attention_bwd_kv_rows,
    block_attention_bwd,
)
from .fp8_fp64 import (  # noqa: F401
    E4M3_MAX,
    DequantView,
    attention_fp8,
    attention_fp8_rows,
    dequantize_blocks,
    e4m3_decode,
    e4m3_encode,
    quantize_blocks,
)
