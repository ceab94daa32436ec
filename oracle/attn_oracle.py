"""fp64 CPU oracle of the attention sublayer that precedes (and, after pruning,
consumes) the pruned MLP block of Representation Shift.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library.

Source: "Representation Shift: Unifying Token Compression with FlashAttention"
(arXiv 2508.00367v1, ICCV 2025).

What it computes for x [L, C] (one sample's tokens), in float64 throughout:

1. u = LN(x)                                   -- Eq. (5)
2. [Q, K, V] = u W_qkv^T + b_qkv               -- Eq. (1), "[Q,K,V] = xW"
3. per head h (columns h*d .. h*d+d-1 of each of Q, K, V, d = C / heads):
   O_h = Softmax(Q_h K_h^T / sqrt(d)) V_h      -- Eq. (1); the softmax runs over
                                                  the keys (each row sums to 1)
4. a = concat_h(O_h) W_o^T + b_o = SA(LN(x))    -- the sublayer output
5. x' = x + a                                  -- Eq. (5)
6. s_t = D(SA(LN(x_t)), x_t)                   -- the representation shift through
                                                  the attention, §3.3 "Operation
                                                  choice" case (i)

Readings where the pages are silent (each also listed in the design notes):
* Eq. (1) is written single-headed with no output projection and scale 1/sqrt(C).
  The models the pages run (DeiT, UMT) use multi-head attention with a bias on
  the QKV projection, an output projection W_o, b_o, and the scale 1/sqrt(d) of
  the head width d = C / heads. With heads = 1, W_o = I and zero biases this is
  Eq. (1) literally (d = C).
* Q, K, V occupy the QKV projection's output columns [0, C), [C, 2C), [2C, 3C);
  head h owns columns h*d .. h*d+d-1 of each (the nn.Linear(C, 3C) layout of
  these models); the heads' outputs are concatenated in head order.
* The LayerNorm is the one of the MLP sublayer (biased variance, eps = 1e-6).
* Pruning after this sublayer by its shift keeps rows of x' with the same rule
  as the MLP block (CLS first and never ranked, ties to the lower index).

Pins (tests/attn_pins.py): a hand-worked two-token case whose softmax weights
are 3/4 and 1/4, uniform attention when the keys carry no information, the
softmax's indifference to a key bias, one-token and two-head closed forms, the
convex-hull property of attention rows, permutation equivariance, and the zero
sublayer (W_o = 0) whose shift is ||x||.
"""
from __future__ import annotations

import numpy as np

from oracle import rs_oracle


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Softmax over the last axis (the keys), shifted by the row maximum."""
    z = S - S.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def attention_core(qkv: np.ndarray, heads: int) -> np.ndarray:
    """Eq. (1) per head on one sample's QKV projection qkv [L, 3C]: the softmax
    attention of every head, concatenated in head order, [L, C]."""
    L, C3 = qkv.shape
    C = C3 // 3
    if C3 != 3 * C or C % heads:
        raise ValueError("qkv must be [L, 3C] with C a multiple of heads")
    d = C // heads
    out = np.empty((L, C))
    for h in range(heads):
        q = qkv[:, h * d:(h + 1) * d]
        k = qkv[:, C + h * d:C + (h + 1) * d]
        v = qkv[:, 2 * C + h * d:2 * C + (h + 1) * d]
        out[:, h * d:(h + 1) * d] = softmax_rows(q @ k.T / np.sqrt(d)) @ v
    return out


def self_attention(u: np.ndarray, Wqkv, bqkv, heads: int) -> np.ndarray:
    """Multi-head form of Eq. (1) for one sample u [L, C]: [Q, K, V] = u W_qkv^T +
    b_qkv, then attention_core."""
    return attention_core(rs_oracle.fc(u, Wqkv, bqkv), heads)


def attn_sublayer(x: np.ndarray, Wqkv, bqkv, Wo, bo, gamma, beta, heads: int,
                  eps: float = rs_oracle.EPS, metric: str = "l2"):
    """Eq. (5) for one sample x [L, C]: returns (a = SA(LN(x)), x' = x + a, s)."""
    u = rs_oracle.layer_norm(x, gamma, beta, eps)
    a = rs_oracle.fc(self_attention(u, Wqkv, bqkv, heads), Wo, bo)
    xp = x + a
    s = rs_oracle.shift_score(a, x, metric)
    return a, xp, s


def attn_forward(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads: int, keep_k: int | None = None,
                 eps: float = rs_oracle.EPS, metric: str = "l2", cls: bool = True):
    """The attention sublayer over x [B, L, C]; with keep_k, pruning by its shift.

    Returns (x' [B, L, C], scores [B, L]) when keep_k is None, else
    (x'_kept [B, n, C], kept_idx [B, n], scores [B, L], x' [B, L, C]) with n = 1 + k
    (CLS kept) or k.
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    xp = np.empty_like(x)
    s = np.empty((B, L))
    for b in range(B):
        _, xp[b], s[b] = attn_sublayer(x[b], Wqkv, bqkv, Wo, bo, gamma, beta, heads, eps, metric)
    if keep_k is None:
        return xp, s
    kept = np.stack([rs_oracle.select_topk(s[b], keep_k, cls) for b in range(B)])
    xk = np.stack([rs_oracle.gather(xp[b], kept[b]) for b in range(B)])
    return xk, kept, s, xp
