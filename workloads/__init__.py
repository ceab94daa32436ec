"""Seeded synthetic inputs for the pruned-MLP block.

This module only draws random numbers and lays out foreground tokens. It holds
none of the method's arithmetic, so both the CUDA path and the fp64 oracle can
take their inputs from it without sharing any of the computation.

The shapes follow the ViT/video-transformer settings of "Representation Shift:
Unifying Token Compression with FlashAttention" (§3.1: N = HW/P^2 patch tokens
of width C; §4.1 UMT video tokens; §4.2 DeiT). Values are synthetic stand-ins
for ImageNet / MSRVTT activations, which are not available here:

* x' ~ N(0, 1); "foreground" patch rows scaled by 3 (CLS is never scaled);
* weights ~ N(0, 0.02) truncated at +-2 sigma by resampling; biases ~ N(0, 0.01);
* LayerNorm gamma = 1 + N(0, 0.05), beta ~ N(0, 0.02);
* everything drawn in fp32 from one CPU ``torch.Generator`` and rounded to
  bf16 exactly once.

Draw order for a stage-0 block with seed ``s``: x, the foreground layout, W1,
b1, W2, b2, gamma, beta, all from ``Generator(s)``. Later stages of a chained
workload draw only their weights, from ``Generator(s + stage)``; their input is
the previous stage's compacted output.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Tuple

import torch

GRID = 14  # 224 / 16 patches per side (DeiT and UMT both use 16x16 patches)


@dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the pruned-MLP block."""

    name: str
    B: int
    L: int
    C: int
    H: int
    keep_k: Tuple[int, ...]  # patch tokens kept at each stage (one entry per stage)
    foreground: str  # "rows40" | "square" | "video_square"
    description: str = ""

    @property
    def stages(self) -> int:
        return len(self.keep_k)

    def stage_L(self, stage: int) -> int:
        """Token count (CLS + patches) entering ``stage``."""
        return self.L if stage == 0 else 1 + self.keep_k[stage - 1]

    def tokens(self, stage: int = 0) -> int:
        return self.B * self.stage_L(stage)

    def flops(self, stage: int = 0) -> float:
        """fc1 + fc2 multiply-adds x2: 4*C*H per token."""
        return 4.0 * self.C * self.H * self.tokens(stage)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_deit_t", B=2, L=197, C=192, H=768, keep_k=(137,), foreground="rows40",
                 description="DeiT-T-shaped block, 40 random foreground rows per sample"),
        Workload("deit_s", B=256, L=197, C=384, H=1536, keep_k=(137,), foreground="square",
                 description="DeiT-S-shaped block, 6x6..10x10 foreground square per sample"),
        Workload("deit_b", B=256, L=197, C=768, H=3072, keep_k=(118,), foreground="square",
                 description="DeiT-B-shaped block, keep ~60% of patches"),
        Workload("umt_b", B=32, L=1569, C=768, H=3072, keep_k=(784,), foreground="video_square",
                 description="UMT-B-shaped video block, 8 frames x 196 patches + CLS, keep 50%"),
        Workload("umt_l", B=16, L=1569, C=1024, H=4096, keep_k=(1097, 767, 536),
                 foreground="video_square",
                 description="UMT-L-shaped 3-stage chain, 70% of patches kept per stage"),
    ]
}


@dataclass
class BlockWeights:
    W1: torch.Tensor  # [H, C] bf16
    b1: torch.Tensor  # [H]    bf16
    W2: torch.Tensor  # [C, H] bf16
    b2: torch.Tensor  # [C]    bf16
    gamma: torch.Tensor  # [C] bf16
    beta: torch.Tensor  # [C] bf16


@dataclass
class BlockInputs:
    x: torch.Tensor  # [B, L, C] bf16 (the attention sublayer's output x')
    foreground: torch.Tensor  # [B, L] bool
    weights: List[BlockWeights] = field(default_factory=list)  # one per stage


def _trunc_normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    """N(0, std) truncated at +-2 std by redrawing the outliers."""
    w = torch.randn(shape, generator=g) * std
    while True:
        bad = w.abs() > 2.0 * std
        n = int(bad.sum())
        if n == 0:
            return w
        w[bad] = torch.randn(n, generator=g) * std


def foreground_layout(g: torch.Generator, B: int, L: int, kind: str) -> torch.Tensor:
    """Boolean [B, L] mask of the rows scaled x3. Token 0 (CLS) is never foreground."""
    fg = torch.zeros(B, L, dtype=torch.bool)
    for b in range(B):
        if kind == "rows40":
            idx = torch.randperm(L - 1, generator=g)[:40] + 1
            fg[b, idx] = True
        elif kind == "square":
            side = int(torch.randint(6, 11, (1,), generator=g))
            r0 = int(torch.randint(0, GRID - side + 1, (1,), generator=g))
            c0 = int(torch.randint(0, GRID - side + 1, (1,), generator=g))
            for r in range(r0, r0 + side):
                for c in range(c0, c0 + side):
                    fg[b, 1 + GRID * r + c] = True
        elif kind == "video_square":
            frames = (L - 1) // (GRID * GRID)
            side, hi = 8, GRID - 8  # start uniform in [0, 6]^2
            r = int(torch.randint(0, hi + 1, (1,), generator=g))
            c = int(torch.randint(0, hi + 1, (1,), generator=g))
            for f in range(frames):
                base = 1 + GRID * GRID * f
                for rr in range(r, r + side):
                    for cc in range(c, c + side):
                        fg[b, base + GRID * rr + cc] = True
                dr = int(torch.randint(-1, 2, (1,), generator=g))
                dc = int(torch.randint(-1, 2, (1,), generator=g))
                r = min(max(r + dr, 0), hi)
                c = min(max(c + dc, 0), hi)
        else:
            raise ValueError(f"unknown foreground layout {kind!r}")
    return fg


def draw_weights(g: torch.Generator, C: int, H: int) -> BlockWeights:
    W1 = _trunc_normal(g, (H, C), 0.02)
    b1 = torch.randn(H, generator=g) * 0.01
    W2 = _trunc_normal(g, (C, H), 0.02)
    b2 = torch.randn(C, generator=g) * 0.01
    gamma = 1.0 + torch.randn(C, generator=g) * 0.05
    beta = torch.randn(C, generator=g) * 0.02
    bf = torch.bfloat16
    return BlockWeights(W1.to(bf), b1.to(bf), W2.to(bf), b2.to(bf), gamma.to(bf), beta.to(bf))


def make_inputs(w: Workload, seed: int = 0, batch: int | None = None) -> BlockInputs:
    """All inputs of ``w`` (every stage's weights) as CPU bf16 tensors.

    ``batch`` overrides B (used to draw a smaller batch of the same shape; the
    draws then differ from the full-size batch from x onwards).
    """
    B = w.B if batch is None else batch
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, w.L, w.C, generator=g)
    fg = foreground_layout(g, B, w.L, w.foreground)
    x[fg] *= 3.0
    weights = [draw_weights(g, w.C, w.H)]
    for s in range(1, w.stages):
        gs = torch.Generator().manual_seed(seed + s)
        weights.append(draw_weights(gs, w.C, w.H))
    return BlockInputs(x=x.to(torch.bfloat16), foreground=fg, weights=weights)


def random_block(B: int, L: int, C: int, H: int, seed: int, fg_rows: int = 0) -> BlockInputs:
    """Same value distributions at an arbitrary shape (edge-case and tail tests)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, L, C, generator=g)
    fg = torch.zeros(B, L, dtype=torch.bool)
    if fg_rows and L > 1:
        for b in range(B):
            idx = torch.randperm(L - 1, generator=g)[: min(fg_rows, L - 1)] + 1
            fg[b, idx] = True
    x[fg] *= 3.0
    return BlockInputs(x=x.to(torch.bfloat16), foreground=fg, weights=[draw_weights(g, C, H)])


@dataclass
class AttnWeights:
    """The attention sublayer's parameters (nn.Linear layouts), bf16."""

    Wqkv: torch.Tensor  # [3C, C]
    bqkv: torch.Tensor  # [3C]
    Wo: torch.Tensor    # [C, C]
    bo: torch.Tensor    # [C]
    gamma: torch.Tensor  # [C]
    beta: torch.Tensor   # [C]


def draw_attn_weights(C: int, seed: int, std: float = 0.02) -> AttnWeights:
    """Attention sublayer weights from ``Generator(seed)`` in the order Wqkv, bqkv,
    Wo, bo, gamma, beta: weights N(0, std) truncated at +-2 std (0.02 is the ViT
    initialisation; larger values give peaked softmax rows), biases N(0, 0.01),
    gamma = 1 + N(0, 0.05), beta ~ N(0, 0.02)."""
    g = torch.Generator().manual_seed(seed)
    Wqkv = _trunc_normal(g, (3 * C, C), std)
    bqkv = torch.randn(3 * C, generator=g) * 0.01
    Wo = _trunc_normal(g, (C, C), std)
    bo = torch.randn(C, generator=g) * 0.01
    gamma = 1.0 + torch.randn(C, generator=g) * 0.05
    beta = torch.randn(C, generator=g) * 0.02
    bf = torch.bfloat16
    return AttnWeights(Wqkv.to(bf), bqkv.to(bf), Wo.to(bf), bo.to(bf), gamma.to(bf), beta.to(bf))


def random_qkv(B: int, L: int, heads: int, seed: int, scale: float = 1.0) -> torch.Tensor:
    """bf16 [B, L, 3 * 64 * heads] QKV projection values ~ N(0, scale^2): with head
    width 64 and the 1/8 scaling, scale 1 gives scores of unit spread, scale 3
    nearly one-hot softmax rows."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, L, 3 * 64 * heads, generator=g) * scale).to(torch.bfloat16)


def random_partials(B: int, L: int, P: int, seed: int, ties: bool = False) -> torch.Tensor:
    """fp32 [B*L, P] non-negative per-row partial sums of squares (select-kernel inputs).

    With ``ties`` the values are drawn from a small set so that equal scores occur.
    """
    g = torch.Generator().manual_seed(seed)
    if ties:
        v = torch.randint(0, 8, (B * L, P), generator=g).float() * 0.25
    else:
        v = torch.rand(B * L, P, generator=g) * 4.0
    return v.contiguous()
