"""fp64 CPU oracle of the pruned-MLP block of Representation Shift.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it. It shares no code with the CUDA library.

Source: "Representation Shift: Unifying Token Compression with FlashAttention"
(arXiv 2508.00367v1, ICCV 2025).

What it computes, per sample and per token row x'_t (the attention sublayer's
output), written out literally and in float64 throughout:

1. u   = LN(x')                      -- LayerNorm named in §3.3, Eq. (6)
2. h   = MLP(u) = fc2(GELU(fc1(u)))  -- the MLP of Eq. (6); fc1 -> erf-GELU -> fc2
3. y   = h + x'                      -- the block output x-hat of Eq. (6)
4. s_t = || MLP(LN(x'_t)) - x'_t ||_2 -- the representation shift of Eq. (4) with
                                       F = the MLP (§3.3 "Operation choice", case
                                       (ii)) and D = the L2 distance (§3.3
                                       "Distance metrics", case (i))
5. drop the lowest-s patch tokens, keep CLS plus the k highest (§3.1 pruned set
   x-tilde in R^{(N-r) x C}; §3.2 "dropped the tokens having the lowest k scores")
6. gather the kept rows of y.

Readings where the pages are silent (each also listed in the design notes):
* LN uses the biased variance and eps = 1e-6; a constant row maps to beta.
* GELU is the exact erf form z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)).
* The score compares the MLP output *without* the residual against x' (Eq. (4)
  with F = MLP o LN as §3.3 writes it), i.e. h - x', not y - x'.
* CLS (t = 0) is always kept and never ranked; its score is still reported.
* Ties in s go to the lower token index; kept rows are in ascending index order.

Pins (tests/test_oracle_pins.py): a hand-worked 4-token example checked against
standard-normal table values, closed forms for degenerate weights (zero score),
brute-force loops for the contractions, exhaustive subset search for top-k,
permutation equivariance, CLS always kept, and LayerNorm moments.
"""
from __future__ import annotations

import numpy as np
from scipy.special import erf

EPS = 1e-6


def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = EPS) -> np.ndarray:
    """LN over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta (biased var).

    LayerNorm as applied to x' in Eq. (6), §3.3.
    """
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU, z * Phi(z), with Phi the standard normal CDF."""
    return 0.5 * z * (1.0 + erf(z / np.sqrt(2.0)))


def fc(v: np.ndarray, W: np.ndarray, b: np.ndarray) -> np.ndarray:
    """nn.Linear layout: W is [out, in]; returns v @ W^T + b."""
    return v @ W.T + b


def mlp(u: np.ndarray, W1, b1, W2, b2) -> np.ndarray:
    """MLP of Eq. (6): fc2(GELU(fc1(u)))."""
    return fc(gelu(fc(u, W1, b1)), W2, b2)


def shift_score(h: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Representation shift, Eq. (4) with D = L2 (§3.2): ||F(x) - x||_2 per row."""
    return np.sqrt(((h - x) ** 2).sum(axis=-1))


def sublayer(x: np.ndarray, W1, b1, W2, b2, gamma, beta, eps: float = EPS):
    """Eq. (6) for token rows x = x' [..., C]: returns (h, y, s)."""
    h = mlp(layer_norm(x, gamma, beta, eps), W1, b1, W2, b2)
    y = h + x
    s = shift_score(h, x)
    return h, y, s


def select_topk(s: np.ndarray, k: int) -> np.ndarray:
    """Kept token indices for one sample: [0] ++ ascending(top-k patch tokens by s).

    Patch tokens are t = 1..L-1. They are ordered by decreasing s, equal s by
    increasing t (a stable sort), and the first k are kept. CLS (t = 0) is
    always first and never ranked.
    """
    L = s.shape[0]
    if not 0 <= k <= L - 1:
        raise ValueError("keep_k out of range")
    t = np.arange(1, L)
    order = np.lexsort((t, -s[1:]))  # primary key -s, secondary key t
    kept = np.sort(t[order[:k]])
    return np.concatenate([np.zeros(1, dtype=np.int64), kept]).astype(np.int64)


def gather(y: np.ndarray, kept: np.ndarray) -> np.ndarray:
    """Rows of y at the kept indices, in that order: the pruned set x-tilde (§3.1)."""
    return y[kept]


def block_forward(x, W1, b1, W2, b2, gamma, beta, keep_k: int, eps: float = EPS):
    """The whole path for x [B, L, C] (float64 values of the stored inputs).

    Returns (y_kept [B, 1+k, C], kept_idx [B, 1+k], scores [B, L], y [B, L, C]).
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    _, y, s = sublayer(x.reshape(B * L, C), W1, b1, W2, b2, gamma, beta, eps)
    y = y.reshape(B, L, C)
    s = s.reshape(B, L)
    kept = np.stack([select_topk(s[b], keep_k) for b in range(B)])
    y_kept = np.stack([gather(y[b], kept[b]) for b in range(B)])
    return y_kept, kept, s, y


def finalize_scores_f32(partials: np.ndarray, B: int, L: int) -> np.ndarray:
    """Scores from fp32 per-row partial sums of squares, in fp32.

    s = sqrt(sum_j P[r, j]) with the partials added left to right in fp32 and a
    correctly rounded fp32 square root. Used where an fp32 score decides the
    integer kept set, so that both sides rank the same fp32 keys.
    """
    p = np.asarray(partials, dtype=np.float32).reshape(B * L, -1)
    acc = np.zeros(B * L, dtype=np.float32)
    for j in range(p.shape[1]):
        acc = (acc + p[:, j]).astype(np.float32)
    return np.sqrt(acc).astype(np.float32).reshape(B, L)
