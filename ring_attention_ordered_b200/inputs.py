"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws the inputs that both
the CUDA path and the fp64 oracle consume, so that the two never share code
beyond the data they are given.

Recipe (identical for every workload):

1. ``torch.Generator("cpu").manual_seed(seed)``;
2. draw float32 ``randn`` in the order Q [B, L, Hq, d], K [B, L, Hkv, d],
   V [B, L, Hkv, d] from that one generator;
3. apply the workload's structure in float32: ``k_scale`` multiplies every key
   (sharper softmax peaks), ``sink_offset`` is added to every component of the
   first ``sink_count`` key positions of every KV head (attention-sink rows:
   a few leading tokens that draw a large share of the attention weight);
4. round to bf16 with round-to-nearest-even (``Tensor.to(torch.bfloat16)``).

The backward pass's upstream gradient dO is drawn the same way from a
generator of its own (``make_grad_output``).

The long-context workloads stand in for the pages' Llama-2 / 128K-token runs,
which need trained weights and datasets that are not used here: the shapes
(sequence length, heads, head dim, ring size) are the pages', the values are
synthetic.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    L: int
    d: int
    n_ring: int
    causal: bool
    seed: int
    k_scale: float = 1.0
    sink_count: int = 0
    sink_offset: float = 0.0
    notes: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def block_len(self) -> int:
        return self.L // self.n_ring

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def flops(self) -> float:
        """Algorithmic FLOPs of one forward pass: 4*B*Hq*L^2*d (two GEMMs of
        2*L^2*d each per head), halved under causal masking."""
        f = 4.0 * self.B * self.Hq * self.L * self.L * self.d
        return f / 2 if self.causal else f

    def flops_exact(self) -> float:
        """FLOPs over exactly the (row, key) pairs the mask keeps:
        L(L+1)/2 pairs per head when causal, L^2 otherwise."""
        pairs = self.L * (self.L + 1) / 2 if self.causal else float(self.L) ** 2
        return 4.0 * self.B * self.Hq * pairs * self.d

    def io_bytes(self) -> int:
        """Compulsory HBM traffic: Q, K, V read once (bf16), O written once
        (bf16), LSE written once (fp32)."""
        q = self.B * self.L * self.Hq * self.d * 2
        kv = 2 * self.B * self.L * self.Hkv * self.d * 2
        return q + kv + q + self.B * self.Hq * self.L * 4

    def describe(self) -> str:
        extra = []
        if self.k_scale != 1.0:
            extra.append(f"K x{self.k_scale:g}")
        if self.sink_count:
            extra.append(f"first {self.sink_count} keys {self.sink_offset:+g}")
        return (f"{'causal' if self.causal else 'non-causal'} B={self.B} Hq={self.Hq} "
                f"Hkv={self.Hkv} L={self.L} d={self.d} n_ring={self.n_ring}"
                + (" (" + ", ".join(extra) + ")" if extra else ""))


WORKLOADS = {
    "l512_d64_noncausal": Workload(
        "l512_d64_noncausal", B=1, Hq=1, Hkv=1, L=512, d=64, n_ring=4,
        causal=False, seed=0),
    "l8k_h8_causal": Workload(
        "l8k_h8_causal", B=2, Hq=8, Hkv=8, L=8192, d=128, n_ring=4,
        causal=True, seed=1),
    "l32k_gqa4_causal": Workload(
        "l32k_gqa4_causal", B=1, Hq=32, Hkv=8, L=32768, d=128, n_ring=8,
        causal=True, seed=2, k_scale=2.0),
    "l128k_h32_causal": Workload(
        "l128k_h32_causal", B=1, Hq=32, Hkv=32, L=131072, d=128, n_ring=8,
        causal=True, seed=3),
    "l1m_gqa4_sink_causal": Workload(
        "l1m_gqa4_sink_causal", B=1, Hq=8, Hkv=2, L=1048576, d=128, n_ring=16,
        causal=True, seed=4, sink_count=4, sink_offset=3.0),
}

# The headline workload: causal attention over 128K tokens, 32 heads, d=128,
# eight ring blocks of 16K tokens.
HEADLINE = "l128k_h32_causal"

# Reduced cases for hardware-counter captures: the headline workload with a
# quarter or half of its heads.  Heads are independent and the forward runs
# them one K/V head after another once K and V exceed 96 MiB, so a launch's
# DRAM traffic scales with the head count (the two sizes check that).  With 8
# heads the bf16 K and V are 512 MiB (about 1 GiB on the device); with 16
# heads the FP8 codes of K and V are 512 MiB too (about 3 GiB on the device
# with the bf16 inputs).
PROFILE_WORKLOADS = {
    "l128k_h8_causal": Workload(
        "l128k_h8_causal", B=1, Hq=8, Hkv=8, L=131072, d=128, n_ring=8,
        causal=True, seed=3),
    "l128k_h16_causal": Workload(
        "l128k_h16_causal", B=1, Hq=16, Hkv=16, L=131072, d=128, n_ring=8,
        causal=True, seed=3),
}


def find_workload(name: str) -> Workload:
    """A named workload or reduced profiling case."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    return PROFILE_WORKLOADS[name]


def make_inputs(B: int, Hq: int, Hkv: int, L: int, d: int, seed: int,
                k_scale: float = 1.0, sink_count: int = 0,
                sink_offset: float = 0.0):
    """Draw (q, k, v) as contiguous bf16 CPU tensors following the recipe in
    the module docstring."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = torch.randn((B, L, Hq, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, L, Hkv, d), generator=g, dtype=torch.float32)
    if k_scale != 1.0:
        k.mul_(k_scale)
    if sink_count:
        k[:, :sink_count] += sink_offset
    k = k.to(torch.bfloat16)
    v = torch.randn((B, L, Hkv, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


# Seed offset of the upstream gradient dO, so that it is drawn from a
# generator of its own and never coincides with Q, K or V.
GRAD_SEED_OFFSET = 1_000_003


def make_grad_output(B: int, L: int, Hq: int, d: int, seed: int):
    """The upstream gradient dO of a backward test or benchmark: standard
    normal fp32 [B, L, Hq, d] from ``torch.Generator("cpu")`` seeded with
    ``seed + GRAD_SEED_OFFSET``, rounded to bf16 (nearest even)."""
    g = torch.Generator(device="cpu").manual_seed(int(seed) + GRAD_SEED_OFFSET)
    return torch.randn((B, L, Hq, d), generator=g, dtype=torch.float32).to(torch.bfloat16)


def workload_inputs(w: Workload):
    return make_inputs(w.B, w.Hq, w.Hkv, w.L, w.d, w.seed, w.k_scale,
                       w.sink_count, w.sink_offset)


def sample_rows(w: Workload, n: int, seed: int | None = None):
    """``n`` distinct (b, h, r) query rows drawn uniformly without replacement
    from ``numpy.random.default_rng(seed)`` (default: the workload's seed),
    returned as an int64 array [n, 3]."""
    import numpy as np

    rng = np.random.default_rng(w.seed if seed is None else seed)
    total = w.B * w.Hq * w.L
    flat = rng.choice(total, size=min(n, total), replace=False)
    b = flat // (w.Hq * w.L)
    h = (flat // w.L) % w.Hq
    r = flat % w.L
    return np.stack([b, h, r], axis=1).astype(np.int64)


def sample_rows_per_head(w: Workload, n: int, seed: int | None = None):
    """``n`` distinct rows of every (b, h), each drawn uniformly without
    replacement from one ``numpy.random.default_rng(seed)`` (default: the
    workload's seed) taken in (b, h) order; int64 array [B * Hq * n, 3]."""
    import numpy as np

    rng = np.random.default_rng(w.seed if seed is None else seed)
    out = []
    for b in range(w.B):
        for h in range(w.Hq):
            r = rng.choice(w.L, size=min(n, w.L), replace=False)
            out.append(np.stack([np.full_like(r, b), np.full_like(r, h), r], axis=1))
    return np.concatenate(out).astype(np.int64)
