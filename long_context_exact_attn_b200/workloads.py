"""Seeded synthetic workloads (shapes and input recipes only, no attention math).

This module is shared by the tests, the benchmark and the CPU oracle's
callers.  It holds no arithmetic of the method: it only draws the inputs.

Recipe: ``g = torch.Generator('cpu').manual_seed(seed)``; draw q, k, v in that
order with ``torch.randn([B, H, N, d], generator=g, dtype=float32)``;
multiply q and k by ``qk_scale_up`` (3 for the stress workload, so that the
logits are large and the online-softmax rescale is exercised); round to
bfloat16 (round-to-nearest-even).  Inputs are produced in token order; the
layout permutation is part of the method, not of the inputs.
"""

from dataclasses import dataclass, replace

import torch

CONTIGUOUS = 0
STRIPED = 1
ZIGZAG = 2
LAYOUT_NAMES = {CONTIGUOUS: "contiguous", STRIPED: "striped", ZIGZAG: "zigzag"}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    P: int
    layout: int
    causal: bool
    seed: int
    qk_scale_up: float = 1.0

    @property
    def c(self):
        return self.N // self.P

    @property
    def scale(self):
        return self.d ** -0.5

    @property
    def layout_name(self):
        return LAYOUT_NAMES[self.layout]

    def useful_pairs(self):
        """Unmasked (query, key) pairs per (batch, head)."""
        n = self.N
        return n * (n + 1) // 2 if self.causal else n * n

    def useful_flops(self):
        """4 d per unmasked pair (2 d for Q K^T, 2 d for P V), all heads."""
        return 4 * self.d * self.B * self.H * self.useful_pairs()

    def with_(self, **kw):
        return replace(self, **kw)


# The five workloads of the method's evaluation, by what they are.
TINY = Workload("tiny_noncausal_N256_d64_P4", 1, 1, 256, 64, 4, CONTIGUOUS, False, 0)
RING_8K = Workload("ring_causal_N8192_H16_d128_P8", 1, 16, 8192, 128, 8, CONTIGUOUS, True, 1)
STRIPED_8K = Workload("striped_causal_N8192_H16_d128_P8", 1, 16, 8192, 128, 8, STRIPED, True, 2)
LONG_128K = Workload("striped_causal_N131072_H8_d128_P8", 1, 8, 131072, 128, 8, STRIPED, True, 3)
STRESS_256K = Workload("striped_causal_N262144_H16_d128_P16_qk3x", 1, 16, 262144, 128, 16,
                       STRIPED, True, 4, qk_scale_up=3.0)

ALL = [TINY, RING_8K, STRIPED_8K, LONG_128K, STRESS_256K]
BY_NAME = {w.name: w for w in ALL}


def make_qkv(w: Workload, device="cpu"):
    """q, k, v as bfloat16 [B, H, N, d] tensors, in token order.

    Each tensor is rounded to bfloat16 right after it is drawn, so that the
    float32 copies of the long workloads are never all alive at once."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    shape = [w.B, w.H, w.N, w.d]
    out = []
    for i in range(3):
        t = torch.randn(shape, generator=g, dtype=torch.float32)
        if i < 2 and w.qk_scale_up != 1.0:
            t.mul_(w.qk_scale_up)
        t = t.to(torch.bfloat16)
        out.append(t.to(device) if device != "cpu" else t)
    return tuple(out)


def make_qkv_head(w: Workload, b: int, h: int):
    """Only head (b, h) of ``make_qkv(w)``, as bfloat16 [N, d] tensors, drawn
    without materialising the other heads.

    torch's CPU normal sampler produces the same stream whether a tensor is
    drawn at once or in consecutive pieces whose sizes are multiples of 16
    (checked by the tests), so the heads before (b, h) are drawn one at a
    time and discarded.
    """
    per_head = w.N * w.d
    if per_head % 16:
        raise ValueError("per-head draws must be a multiple of 16 values")
    g = torch.Generator("cpu").manual_seed(w.seed)
    n_heads = w.B * w.H
    idx = b * w.H + h
    out = []
    for _ in range(3):
        for _skip in range(idx):
            torch.randn([per_head], generator=g, dtype=torch.float32)
        out.append(torch.randn([per_head], generator=g, dtype=torch.float32).view(w.N, w.d))
        for _skip in range(n_heads - idx - 1):
            torch.randn([per_head], generator=g, dtype=torch.float32)
    q, k, v = out
    if w.qk_scale_up != 1.0:
        q = q * w.qk_scale_up
        k = k * w.qk_scale_up
    return tuple(t.to(torch.bfloat16) for t in (q, k, v))
