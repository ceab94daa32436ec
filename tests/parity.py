"""Parity rules between the CUDA path and the fp64 oracle.

Tolerances (derived from the arithmetic: bf16 GEMM operands, fp32 accumulation,
a bf16 hidden activation and a bf16 store of y):
* y (every compared row): max|y_gpu - y_ref| / max|y_ref| <= 2e-2, and
  elementwise |y_gpu - y_ref| <= 2e-2 * max(1, |y_ref|);
* scores: |s_gpu - s_ref| <= 1e-2 * max(s_ref, 1e-6) per token;
* kept_idx: bit-exact where the oracle's k-th and (k+1)-th largest patch scores
  differ by at least 1e-3 relative; otherwise the GPU's set must be a valid
  top-k under the oracle's scores within that band (min kept >= max dropped -
  1e-3 * t_k), with CLS first and indices ascending and unique.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

Y_TOL = 2e-2
S_TOL = 1e-2
GAP_TOL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def weights64(w):
    return dict(W1=f64(w.W1), b1=f64(w.b1), W2=f64(w.W2), b2=f64(w.b2),
                gamma=f64(w.gamma), beta=f64(w.beta))


def oracle_block(x_bf16: torch.Tensor, w, keep_k: int, metric: str = "l2", cls: bool = True):
    """Oracle on bf16 CPU inputs [B, L, C]: (y_kept, kept, scores, y) in float64."""
    return oracle.block_forward(f64(x_bf16), keep_k=keep_k, metric=metric, cls=cls,
                                **weights64(w))


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "y") -> float:
    d = np.abs(y_gpu - y_ref)
    scale = max(np.abs(y_ref).max(), 1e-30)
    rel = d.max() / scale
    assert rel <= Y_TOL, f"{what}: max-abs error {d.max():.3e} / max|ref| {scale:.3e} = {rel:.3e}"
    bad = d > Y_TOL * np.maximum(1.0, np.abs(y_ref))
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside 2e-2*max(1,|ref|)"
    return float(rel)


def check_scores(s_gpu: np.ndarray, s_ref: np.ndarray) -> float:
    d = np.abs(s_gpu - s_ref)
    lim = S_TOL * np.maximum(s_ref, 1e-6)
    assert np.all(d <= lim), f"scores: worst {np.max(d / np.maximum(s_ref, 1e-6)):.3e} relative"
    return float(np.max(d / np.maximum(s_ref, 1e-6)))


def check_kept(kept_gpu: np.ndarray, s_ref_row: np.ndarray, kept_ref: np.ndarray, k: int,
               cls: bool = True) -> bool:
    """Returns True when the exact rule applied (False: band rule). With a CLS token
    the list is [0] ++ k ranked patch tokens; without, k ranked tokens of 0..L-1."""
    L = s_ref_row.shape[0]
    first = 1 if cls else 0
    kg = [int(v) for v in kept_gpu]
    assert len(kg) == k + first, (len(kg), k)
    if cls:
        assert kg[0] == 0, kg[:4]
    ranked = kg[first:]
    assert all(kg[i] < kg[i + 1] for i in range(len(kg) - 1)), "kept indices not ascending/unique"
    assert all(first <= t < L for t in ranked)
    if k == 0 or k == L - first:
        assert kg == list(kept_ref)
        return True
    sp = np.sort(s_ref_row[first:])[::-1]
    t_k, t_k1 = sp[k - 1], sp[k]
    if (t_k - t_k1) >= GAP_TOL * t_k:
        assert kg == list(kept_ref), "kept_idx differs where the oracle's gap is >= 1e-3"
        return True
    kept_set = set(ranked)
    dropped = [t for t in range(first, L) if t not in kept_set]
    assert min(s_ref_row[t] for t in ranked) >= max(s_ref_row[t] for t in dropped) - GAP_TOL * t_k
    return False


def check_block(gpu, ref, k: int, samples=None, cls: bool = True) -> dict:
    """gpu = (y_kept, kept_idx, scores) torch tensors (full batch); ref = oracle output on
    the batch rows listed in ``samples`` (all when None)."""
    y_kept_g, kept_g, s_g = (t.detach().cpu() for t in gpu)
    y_kept_r, kept_r, s_r, y_r = ref
    B = y_kept_g.shape[0]
    samples = list(range(B)) if samples is None else list(samples)
    exact = 0
    worst_y = 0.0
    worst_s = check_scores(f64(s_g)[samples], s_r)
    for i, b in enumerate(samples):
        kg = kept_g[b].numpy()
        exact += check_kept(kg, s_r[i], kept_r[i], k, cls)
        if kg.size:  # no kept row at all without CLS and keep_k = 0
            worst_y = max(worst_y, check_y(f64(y_kept_g[b]), y_r[i][kg.astype(np.int64)],
                                           f"y_kept[{b}]"))
    return dict(exact=exact, band=len(samples) - exact, worst_y=worst_y, worst_s=worst_s)
