"""CPU models of where the CUDA kernels round (test infrastructure).

These are NOT the oracle. The oracle (``oracle/``) computes what the paper
defines, in float64 with no intermediate rounding. The functions here take the
same float64 steps but round to bf16 (or compute in fp32) exactly where the
kernels store or convert a value. Tests use them for two things:

* to make an integer decision on the same fp32 keys the kernel ranks
  (``finalize_scores_f32``: the selection kernel adds a row's partial sums left
  to right in fp32), so that kept sets can be compared bit for bit;
* to show that a disagreement between the kernels and the oracle follows from
  the bf16 rounding that the kernels' data layout imposes, and not from a kernel
  error (``attn_sublayer_bf16``): where the sublayer is ill-conditioned in its
  bf16 operands, the model leaves the oracle's tolerance on its own, and the
  kernels are then held to the model.

Every rounding point can be switched off (``rounding=False``), which must give
back the oracle's result to float64 accuracy (tests/test_kernel_model.py): the
model differs from the oracle only where it rounds.

Source of the computation: "Representation Shift: Unifying Token Compression
with FlashAttention", Eq. (1) and Eq. (5) (the attention sublayer), §3.3
"Distance metrics" (the score of each distance).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import rs_oracle

COS_EPS = rs_oracle.COS_EPS  # the cosine distance's denominator floor (a reading of §3.3)


def bf16(a: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even) through fp32, as the kernels convert
    an fp32 value; returned widened to float64."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def finalize_scores_f32(partials: np.ndarray, B: int, L: int, metric: str = "l2") -> np.ndarray:
    """Scores from fp32 per-row partial sums, in fp32 (correctly rounded operations),
    as the selection kernel forms its keys.

    l2:     partials are sums of (h - x)^2 over column groups; s = sqrt(sum_j P[r, j]).
    l1:     partials are sums of |h - x|; s = sum_j P[r, j].
    cosine: partials are triples (sum h.x, sum h.h, sum x.x) per column group;
            s = max(0, 1 - HX / max(sqrt(HH) * sqrt(XX), COS_EPS)) with HX, HH, XX the
            group sums. Floored at 0 so that the fp32 bits order like the values.
    Partials are added left to right (group order).
    """
    f32 = np.float32
    p = np.asarray(partials, dtype=f32).reshape(B * L, -1)

    def rsum(cols):
        acc = np.zeros(B * L, dtype=f32)
        for j in cols:
            acc = (acc + p[:, j]).astype(f32)
        return acc

    if metric == "l2":
        return np.sqrt(rsum(range(p.shape[1]))).astype(f32).reshape(B, L)
    if metric == "l1":
        return rsum(range(p.shape[1])).reshape(B, L)
    if metric == "cosine":
        if p.shape[1] % 3:
            raise ValueError("cosine partials come in triples")
        n = p.shape[1]
        hx, hh, xx = rsum(range(0, n, 3)), rsum(range(1, n, 3)), rsum(range(2, n, 3))
        den = np.maximum((np.sqrt(hh) * np.sqrt(xx)).astype(f32), f32(COS_EPS))
        s = (f32(1.0) - (hx / den).astype(f32)).astype(f32)
        return np.maximum(s, f32(0.0)).reshape(B, L)
    raise ValueError(f"unknown metric {metric!r}")


def folded_projection(x: np.ndarray, W: np.ndarray, b: np.ndarray, gamma: np.ndarray,
                      beta: np.ndarray, rounding: bool = True, eps: float = rs_oracle.EPS):
    """LN(x) W^T + b as the folded-LN GEMM forms it, for x [M, C]:
    Wg = bf16(W * gamma) (the fold's stored weights), G = sum_c Wg, cb = W beta + b,
    z = rstd * (x Wg^T - mean * G) + cb. Without rounding Wg = W * gamma, and z is
    LN(x) W^T + b exactly (in exact arithmetic)."""
    Wg = W * gamma[None, :]
    if rounding:
        Wg = bf16(Wg)
    G = Wg.sum(axis=1)
    cb = W @ beta + b
    mean = x.mean(axis=1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    return rstd * (x @ Wg.T - mean * G[None, :]) + cb[None, :]


def attention_core_bf16(qkv: np.ndarray, heads: int, rounding: bool = True,
                        block: int = 64, rescale_above: float = 8.0) -> np.ndarray:
    """Softmax(Q K^T / sqrt(d)) V per head (d = 64) for one sample's qkv [L, 3C], in
    the order the attention kernel takes its steps: keys in blocks of ``block``;
    per query row a reference maximum m (log2 units) that moves only when a block's
    maximum exceeds it by more than ``rescale_above``; P = 2^(s log2(e)/8 - m) summed
    unrounded into l but rounded to bf16 for the P V product; the result O / l
    rounded to bf16. Without rounding this is the plain softmax attention."""
    L, C3 = qkv.shape
    C = C3 // 3
    d = C // heads
    c = np.log2(np.e) / np.sqrt(d)
    out = np.empty((L, C))
    rnd = bf16 if rounding else (lambda a: a)
    for h in range(heads):
        q = qkv[:, h * d:(h + 1) * d]
        k = qkv[:, C + h * d:C + (h + 1) * d]
        v = qkv[:, 2 * C + h * d:2 * C + (h + 1) * d]
        m = np.full(L, -np.inf)
        lsum = np.zeros(L)
        o = np.zeros((L, d))
        for j0 in range(0, L, block):
            s = (q @ k[j0:j0 + block].T) * c
            m_blk = s.max(axis=1)
            move = m_blk > m + rescale_above
            m_new = np.where(move, m_blk, m)
            alpha = np.where(move, np.exp2(np.where(np.isinf(m), -np.inf, m - m_new)), 1.0)
            p = np.exp2(s - m_new[:, None])
            lsum = lsum * alpha + p.sum(axis=1)
            o = o * alpha[:, None] + rnd(p) @ v[j0:j0 + block]
            m = m_new
        out[:, h * d:(h + 1) * d] = rnd(o / lsum[:, None])
    return out


def attn_sublayer_bf16(x: np.ndarray, Wqkv, bqkv, Wo, bo, gamma, beta, heads: int,
                       rounding: bool = True) -> np.ndarray:
    """x' = x + SA(LN(x)) W_o^T + b_o (Eq. (5)) for x [B, L, C] with the kernels'
    rounding points: the folded-LN QKV projection (bf16 folded weights) stored as
    bf16, the attention core of ``attention_core_bf16``, the output projection on
    the bf16 attention output, and x' stored as bf16."""
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    rnd = bf16 if rounding else (lambda a: a)
    out = np.empty_like(x)
    for b in range(B):
        qkv = rnd(folded_projection(x[b], Wqkv, bqkv, gamma, beta, rounding))
        a = attention_core_bf16(qkv, heads, rounding)
        out[b] = rnd(x[b] + a @ Wo.T + bo[None, :])
    return out
