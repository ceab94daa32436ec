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
                                       "Distance metrics", case (i)); the L1 and
                                       cosine distances (cases (ii), (iii)) too
5. drop the lowest-s patch tokens, keep CLS plus the k highest (§3.1 pruned set
   x-tilde in R^{(N-r) x C}; §3.2 "dropped the tokens having the lowest k scores")
6. gather the kept rows of y.

Readings where the pages are silent (each also listed in the design notes):
* LN uses the biased variance and eps = 1e-6; a constant row maps to beta.
* GELU is the exact erf form z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)).
* The score compares the MLP output *without* the residual against x' (Eq. (4)
  with F = MLP o LN as §3.3 writes it), i.e. h - x', not y - x'.
* CLS (t = 0) is always kept and never ranked; its score is still reported.
  Without a CLS token (cls=False) all L tokens are ranked.
* The cosine distance floors ||h|| ||x'|| at 1e-8; in fp32 it is floored at 0.
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


METRICS = ("l2", "l1", "cosine")
COS_EPS = 1e-8  # floor of ||h|| ||x|| in the cosine distance (the pages give none)


def shift_score(h: np.ndarray, x: np.ndarray, metric: str = "l2") -> np.ndarray:
    """Representation shift, Eq. (4), D(F(x'), x') per row with F(x') = h, the MLP output
    (§3.3 "Operation choice" (ii)) and D one of §3.3 "Distance metrics":
      (i)   l2:     ||h - x||_2
      (ii)  l1:     ||h - x||_1
      (iii) cosine: 1 - h.x / (||h|| ||x||), the denominator floored at COS_EPS.
    """
    if metric == "l2":
        return np.sqrt(((h - x) ** 2).sum(axis=-1))
    if metric == "l1":
        return np.abs(h - x).sum(axis=-1)
    if metric == "cosine":
        dot = (h * x).sum(axis=-1)
        den = np.sqrt((h * h).sum(axis=-1)) * np.sqrt((x * x).sum(axis=-1))
        return 1.0 - dot / np.maximum(den, COS_EPS)
    raise ValueError(f"unknown metric {metric!r}")


def sublayer(x: np.ndarray, W1, b1, W2, b2, gamma, beta, eps: float = EPS, metric: str = "l2"):
    """Eq. (6) for token rows x = x' [..., C]: returns (h, y, s)."""
    h = mlp(layer_norm(x, gamma, beta, eps), W1, b1, W2, b2)
    y = h + x
    s = shift_score(h, x, metric)
    return h, y, s


def select_topk(s: np.ndarray, k: int, cls: bool = True) -> np.ndarray:
    """Kept token indices for one sample.

    With a CLS token (cls=True): [0] ++ ascending(top-k patch tokens by s); patch
    tokens are t = 1..L-1 and CLS (t = 0) is always first and never ranked.
    Without (cls=False, a video sequence of patch tokens only): ascending(top-k of all
    L tokens). Ranking: decreasing s, equal s by increasing t (a stable sort).
    """
    L = s.shape[0]
    first = 1 if cls else 0
    if not 0 <= k <= L - first:
        raise ValueError("keep_k out of range")
    t = np.arange(first, L)
    order = np.lexsort((t, -s[first:]))  # primary key -s, secondary key t
    kept = np.sort(t[order[:k]]).astype(np.int64)
    if cls:
        return np.concatenate([np.zeros(1, dtype=np.int64), kept])
    return kept


def gather(y: np.ndarray, kept: np.ndarray) -> np.ndarray:
    """Rows of y at the kept indices, in that order: the pruned set x-tilde (§3.1)."""
    return y[kept]


def block_forward(x, W1, b1, W2, b2, gamma, beta, keep_k: int, eps: float = EPS,
                  metric: str = "l2", cls: bool = True):
    """The whole path for x [B, L, C] (float64 values of the stored inputs).

    Returns (y_kept [B, n, C], kept_idx [B, n], scores [B, L], y [B, L, C]) with
    n = 1 + k (CLS kept) or k (cls=False).
    """
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    _, y, s = sublayer(x.reshape(B * L, C), W1, b1, W2, b2, gamma, beta, eps, metric)
    y = y.reshape(B, L, C)
    s = s.reshape(B, L)
    kept = np.stack([select_topk(s[b], keep_k, cls) for b in range(B)])
    y_kept = np.stack([gather(y[b], kept[b]) for b in range(B)])
    return y_kept, kept, s, y


def block_shift_forward(x_in, x, W1, b1, W2, b2, gamma, beta, keep_k: int, eps: float = EPS,
                        metric: str = "l2", cls: bool = True):
    """Pruning on the shift through the entire attention block, §3.3 "Operation
    choice" case (iii): s = D(x-hat, x_in), with x-hat = y = x' + MLP(LN(x')) the
    block output (Eq. (6)) and x_in the block input that Eq. (5) started from.
    x_in, x (= x') [B, L, C]; returns what block_forward returns."""
    x_in = np.asarray(x_in, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    _, y, _ = sublayer(x.reshape(B * L, C), W1, b1, W2, b2, gamma, beta, eps, metric)
    s = shift_score(y, x_in.reshape(B * L, C), metric).reshape(B, L)
    y = y.reshape(B, L, C)
    kept = np.stack([select_topk(s[b], keep_k, cls) for b in range(B)])
    y_kept = np.stack([gather(y[b], kept[b]) for b in range(B)])
    return y_kept, kept, s, y
