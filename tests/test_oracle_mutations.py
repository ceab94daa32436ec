"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin fails.

Each mutation replaces one oracle function with a wrong variant: a dropped
term, a wrong sign, a transposed operand, a wrong normalisation, a reversed
tie rule. The pins must reject every one of them.
"""
import numpy as np
import pytest
from scipy.special import erf

import oracle.rs_oracle as rs_oracle
from oracle_pins import ALL_PINS

orig = {n: getattr(rs_oracle, n) for n in
        ["layer_norm", "gelu", "fc", "mlp", "shift_score", "select_topk", "gather", "sublayer"]}


def _ln_unbiased(x, gamma, beta, eps=rs_oracle.EPS):
    mu = x.mean(axis=-1, keepdims=True)
    var = x.var(axis=-1, ddof=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def _ln_no_beta(x, gamma, beta, eps=rs_oracle.EPS):
    return orig["layer_norm"](x, gamma, np.zeros_like(beta), eps)


def _ln_no_eps(x, gamma, beta, eps=rs_oracle.EPS):
    return orig["layer_norm"](x, gamma, beta, 0.0)


def _ln_no_gamma(x, gamma, beta, eps=rs_oracle.EPS):
    return orig["layer_norm"](x, np.ones_like(gamma), beta, eps)


def _gelu_no_sqrt2(z):
    return 0.5 * z * (1.0 + erf(z))


def _gelu_tanh(z):
    return 0.5 * z * (1.0 + np.tanh(np.sqrt(2 / np.pi) * (z + 0.044715 * z ** 3)))


def _fc_transposed(v, W, b):
    return v @ W + b  # weight read as [in, out]: wrong for nn.Linear's [out, in]


def _fc_no_bias(v, W, b):
    return v @ W.T


def _mlp_relu(u, W1, b1, W2, b2):
    return rs_oracle.fc(np.maximum(rs_oracle.fc(u, W1, b1), 0), W2, b2)


def _mlp_no_act(u, W1, b1, W2, b2):
    return rs_oracle.fc(rs_oracle.fc(u, W1, b1), W2, b2)


# Mutants of one metric (or of the CLS mode) delegate every other case to the
# original function, so that a pin has to catch the planted mistake itself.
def _for_metric(metric, bad):
    def f(h, x, m="l2"):
        return bad(h, x) if m == metric else orig["shift_score"](h, x, m)
    return f


def _for_cls(bad):
    def f(s, k, cls=True):
        return bad(s, k) if cls else orig["select_topk"](s, k, cls)
    return f


def _score_plus(h, x):
    return np.sqrt(((h + x) ** 2).sum(axis=-1))


def _score_residual(h, x):  # ||(h + x) - x|| = ||h||
    return np.sqrt((h ** 2).sum(axis=-1))


def _score_squared(h, x):
    return ((h - x) ** 2).sum(axis=-1)


def _score_l1(h, x):
    return np.abs(h - x).sum(axis=-1)


def _l1_no_abs(h, x):
    return (h - x).sum(axis=-1)


def _cos_similarity(h, x):  # the similarity, not the distance
    return (h * x).sum(-1) / (np.linalg.norm(h, axis=-1) * np.linalg.norm(x, axis=-1))


def _cos_of_output(h, x):  # angle between y = h + x and x
    y = h + x
    return 1 - (y * x).sum(-1) / (np.linalg.norm(y, axis=-1) * np.linalg.norm(x, axis=-1))


def _cos_unnormalised(h, x):
    return 1 - (h * x).sum(-1)


def _select_ties_high(s, k):
    L = s.shape[0]
    t = np.arange(1, L)
    order = np.lexsort((-t, -s[1:]))
    return np.concatenate([[0], np.sort(t[order[:k]])]).astype(np.int64)


def _select_lowest(s, k):
    L = s.shape[0]
    t = np.arange(1, L)
    order = np.lexsort((t, s[1:]))
    return np.concatenate([[0], np.sort(t[order[:k]])]).astype(np.int64)


def _select_rank_cls(s, k):
    L = s.shape[0]
    t = np.arange(0, L)
    order = np.lexsort((t, -s))
    return np.sort(t[order[: k + 1]]).astype(np.int64)


def _select_unsorted(s, k):
    L = s.shape[0]
    t = np.arange(1, L)
    order = np.lexsort((t, -s[1:]))
    return np.concatenate([[0], t[order[:k]]]).astype(np.int64)


def _no_cls_still_keeps_cls(s, k, cls=True):
    return orig["select_topk"](s, k, True) if not cls or True else None


def _no_cls_skips_t0(s, k, cls=True):
    if cls:
        return orig["select_topk"](s, k, True)
    if k > len(s) - 1:
        k = len(s) - 1
    return orig["select_topk"](s, k, True)[1:]


def _gather_shift(y, kept):
    return y[np.minimum(kept + 1, y.shape[0] - 1)]


def _sublayer_score_after_residual(x, W1, b1, W2, b2, gamma, beta, eps=rs_oracle.EPS,
                                   metric="l2"):
    h = rs_oracle.mlp(rs_oracle.layer_norm(x, gamma, beta, eps), W1, b1, W2, b2)
    y = h + x
    return h, y, rs_oracle.shift_score(y, x, metric)


def _sublayer_no_residual(x, W1, b1, W2, b2, gamma, beta, eps=rs_oracle.EPS, metric="l2"):
    h = rs_oracle.mlp(rs_oracle.layer_norm(x, gamma, beta, eps), W1, b1, W2, b2)
    return h, h, rs_oracle.shift_score(h, x, metric)


def _block_shift_vs_x_prime(x_in, x, W1, b1, W2, b2, gamma, beta, keep_k, eps=rs_oracle.EPS,
                            metric="l2", cls=True):
    # compares y with x' instead of the block input: the MLP shift of case (ii) in disguise
    return _orig_block_shift(x, x, W1, b1, W2, b2, gamma, beta, keep_k, eps, metric, cls)


def _block_shift_of_h(x_in, x, W1, b1, W2, b2, gamma, beta, keep_k, eps=rs_oracle.EPS,
                      metric="l2", cls=True):
    # compares the MLP output h (not the block output y) with the block input
    x_in = np.asarray(x_in, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    h, y, _ = rs_oracle.sublayer(x.reshape(B * L, C), W1, b1, W2, b2, gamma, beta, eps, metric)
    s = rs_oracle.shift_score(h, x_in.reshape(B * L, C), metric).reshape(B, L)
    y = y.reshape(B, L, C)
    kept = np.stack([rs_oracle.select_topk(s[b], keep_k, cls) for b in range(B)])
    return np.stack([y[b][kept[b]] for b in range(B)]), kept, s, y


_orig_block_shift = rs_oracle.block_shift_forward

MUTATIONS = {
    "block_shift_against_x_prime": ("block_shift_forward", _block_shift_vs_x_prime),
    "block_shift_of_mlp_output": ("block_shift_forward", _block_shift_of_h),
    "ln_unbiased_var": ("layer_norm", _ln_unbiased),
    "ln_drops_beta": ("layer_norm", _ln_no_beta),
    "ln_drops_gamma": ("layer_norm", _ln_no_gamma),
    "ln_drops_eps": ("layer_norm", _ln_no_eps),
    "gelu_erf_without_sqrt2": ("gelu", _gelu_no_sqrt2),
    "gelu_tanh_approx": ("gelu", _gelu_tanh),
    "fc_transposed_weight": ("fc", _fc_transposed),
    "fc_drops_bias": ("fc", _fc_no_bias),
    "mlp_relu": ("mlp", _mlp_relu),
    "mlp_no_activation": ("mlp", _mlp_no_act),
    "score_plus_sign": ("shift_score", _for_metric("l2", _score_plus)),
    "score_squared": ("shift_score", _for_metric("l2", _score_squared)),
    "score_l1": ("shift_score", _for_metric("l2", _score_l1)),
    "score_of_h_only": ("shift_score", _for_metric("l2", _score_residual)),
    "l1_squared": ("shift_score", _for_metric("l1", _score_squared)),
    "l1_without_abs": ("shift_score", _for_metric("l1", _l1_no_abs)),
    "cosine_similarity_not_distance": ("shift_score", _for_metric("cosine", _cos_similarity)),
    "cosine_of_block_output": ("shift_score", _for_metric("cosine", _cos_of_output)),
    "cosine_unnormalised": ("shift_score", _for_metric("cosine", _cos_unnormalised)),
    "select_ties_to_higher_index": ("select_topk", _for_cls(_select_ties_high)),
    "select_keeps_lowest": ("select_topk", _for_cls(_select_lowest)),
    "select_ranks_cls": ("select_topk", _for_cls(_select_rank_cls)),
    "select_unsorted_output": ("select_topk", _for_cls(_select_unsorted)),
    "no_cls_still_keeps_cls": ("select_topk", _no_cls_still_keeps_cls),
    "no_cls_never_keeps_t0": ("select_topk", _no_cls_skips_t0),
    "gather_off_by_one": ("gather", _gather_shift),
    "score_after_residual": ("sublayer", _sublayer_score_after_residual),
    "no_residual": ("sublayer", _sublayer_no_residual),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    fn_name, bad = MUTATIONS[name]
    monkeypatch.setattr(rs_oracle, fn_name, bad)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(rs_oracle)
        except Exception as e:  # AssertionError or a shape error from a bad operand
            caught.append((pin.__name__, type(e).__name__))
    assert caught, f"no pin caught mutation {name}"
