"""fp64 CPU oracle of a ViT encoder with representation-shift pruning between layers.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library.

Source: "Representation Shift: Unifying Token Compression with FlashAttention"
(arXiv 2508.00367v1, ICCV 2025). Each layer is Eq. (5) then Eq. (6); after the
MLP of a pruning layer the tokens with the lowest shift ||MLP(LN(x')) - x'||_2
are dropped (§3.2, §3.3 case (ii) with the L2 distance), CLS kept. §4.2 prunes
20% of the tokens after layers [1, 4, 7] of DeiT.

Reading where the pages are silent: "20% of the tokens" is taken of the patch
tokens entering the layer, rounded to the nearest integer (196 -> keep 157 ->
126 -> 101 for DeiT at 224^2).
"""
from __future__ import annotations

import numpy as np

from oracle import attn_oracle, rs_oracle


def keep_after_pruning(patches: int, ratio: float = 0.2) -> int:
    """Patch tokens kept when `ratio` of `patches` is pruned (nearest integer)."""
    return patches - int(np.floor(ratio * patches + 0.5))


def deit_schedule(depth: int = 12, L: int = 197, layers=(1, 4, 7), ratio: float = 0.2):
    """keep[l] for every layer: patch tokens kept after layer l, or -1 (no pruning)."""
    keep = [-1] * depth
    patches = L - 1
    for l in layers:
        patches = keep_after_pruning(patches, ratio)
        keep[l] = patches
    return keep


def encoder_forward(x, layers, keep, heads: int, eps: float = rs_oracle.EPS):
    """x [B, L, C]; layers[l] a dict with Wqkv, bqkv, Wo, bo, gamma1, beta1, W1, b1, W2,
    b2, gamma2, beta2; keep[l] patch tokens kept after layer l or < 0. Returns the
    last layer's output [B, L_out, C] and the kept indices of every pruning layer."""
    cur = np.asarray(x, dtype=np.float64)
    kept_all = []
    for w, k in zip(layers, keep):
        xp, _ = attn_oracle.attn_forward(cur, w["Wqkv"], w["bqkv"], w["Wo"], w["bo"],
                                         w["gamma1"], w["beta1"], heads, eps=eps)
        mlp = dict(W1=w["W1"], b1=w["b1"], W2=w["W2"], b2=w["b2"], gamma=w["gamma2"],
                   beta=w["beta2"])
        if k >= 0:
            cur, kept, _, _ = rs_oracle.block_forward(xp, keep_k=k, eps=eps, **mlp)
            kept_all.append(kept)
        else:
            B, L, C = xp.shape
            _, y, _ = rs_oracle.sublayer(xp.reshape(B * L, C), eps=eps, **mlp)
            cur = y.reshape(B, L, C)
    return cur, kept_all
