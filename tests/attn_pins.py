"""Pins of the attention oracle to facts that do not come from the oracle itself.

Each ``pin_*`` takes the attention oracle *module* and raises AssertionError when
it disagrees with the fact; calls go through the module's attributes so that a
test can plant a mistake in one function and check that a pin catches it.

Sources of truth:
* two hand-worked cases (tests/golden/attn_two_token.json): the sublayer of
  Eq. (5) whose softmax weights are 3/4 and 1/4, and a two-head attention core;
* closed forms: uniform attention when the keys carry no information, one token
  (softmax weight 1), the zero sublayer (W_o = 0) whose shift is the size of x;
* invariants: a key bias cancels in the softmax, attention rows are convex
  combinations of the value rows, permutation equivariance over tokens, samples
  do not mix.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import rs_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "attn_two_token.json")) as f:
        return json.load(f)


def _weights(rng, C, scale=0.3):
    return dict(Wqkv=rng.normal(0, scale, (3 * C, C)), bqkv=rng.normal(0, 0.1, 3 * C),
                Wo=rng.normal(0, scale, (C, C)), bo=rng.normal(0, 0.1, C),
                gamma=1 + rng.normal(0, 0.2, C), beta=rng.normal(0, 0.1, C))


def _run(o, x, w, heads, metric="l2"):
    return o.attn_sublayer(x, w["Wqkv"], w["bqkv"], w["Wo"], w["bo"], w["gamma"], w["beta"],
                           heads, metric=metric)


def pin_attn_hand_sublayer(o):
    """The two-token sublayer: weights 3/4, 1/4; x' and the three shifts. Against the
    hand values (eps = 0) within 1e-5, and exactly against the same derivation
    carried out with eps = 1e-6 (each LN row scaled by f = 1/sqrt(1 + eps))."""
    g = _golden()["sublayer_case"]
    x = np.array(g["x"])
    alpha = math.sqrt(math.log(3.0) / (2.0 * math.sqrt(2.0)))
    eye = np.eye(2)
    w = dict(Wqkv=np.vstack([alpha * eye, alpha * eye, eye]), bqkv=np.zeros(6), Wo=eye,
             bo=np.zeros(2), gamma=np.ones(2), beta=np.zeros(2))
    f = 1.0 / math.sqrt(1.0 + rs_oracle.EPS)
    # with eps: scores +-f^2 ln(3)/2, so w00 - w01 = tanh(f^2 ln(3) / 2), and a_0 = f (w00 - w01) x_0
    ft = f * math.tanh(f * f * math.log(3.0) / 2.0)   # a_t = ft x_t
    exact = {"l2": abs(1.0 - ft) * math.sqrt(2.0), "l1": 2.0 * abs(1.0 - ft), "cosine": 0.0}
    for metric, key in (("l2", "shift_l2"), ("l1", "shift_l1"), ("cosine", "shift_cosine")):
        a, xp, s = _run(o, x, w, 1, metric)
        assert np.allclose(a, g["a"], atol=1e-5, rtol=0), a
        assert np.allclose(xp, g["x_out"], atol=1e-5, rtol=0), xp
        assert np.allclose(s, g[key], atol=1e-5, rtol=0), (metric, s)
        assert np.allclose(xp, (1.0 + ft) * x, atol=1e-12, rtol=0), (xp, ft)
        assert np.allclose(s, exact[metric], atol=1e-12, rtol=0), (metric, s, exact[metric])


def pin_attn_hand_core(o):
    """The two-head attention core with one uniform and one 3/4-1/4 head."""
    g = _golden()["core_case"]
    b = math.sqrt(math.sqrt(2.0) * math.log(3.0) / 2.0)
    qkv = np.zeros((2, 12))
    qkv[0, 2:4] = [b, 0.0]   # q, head 1
    qkv[1, 2:4] = [-b, 0.0]
    qkv[0, 6:8] = [b, 0.0]   # k, head 1
    qkv[1, 6:8] = [-b, 0.0]
    qkv[:, 8:10] = g["v_head0"]
    qkv[:, 10:12] = g["v_head1"]
    out = o.attention_core(qkv, 2)
    assert np.allclose(out, g["out"], atol=1e-12, rtol=0), out


def pin_attn_uniform_keys(o):
    """W_k = 0: every score of a row is the same (q . b_k), so every token gets the
    mean of the value rows, whatever the key bias and the queries."""
    rng = np.random.default_rng(31)
    C, L, heads = 8, 7, 2
    w = _weights(rng, C)
    w["Wqkv"][C:2 * C] = 0.0
    x = rng.normal(0, 1, (L, C))
    a, xp, _ = _run(o, x, w, heads)
    u = rs_oracle.layer_norm(x, w["gamma"], w["beta"])
    v = u @ w["Wqkv"][2 * C:].T + w["bqkv"][2 * C:]
    want = v.mean(axis=0) @ w["Wo"].T + w["bo"]
    assert np.allclose(a, np.broadcast_to(want, a.shape), atol=1e-12, rtol=0)
    assert np.array_equal(xp, x + a)


def pin_attn_key_bias(o):
    """A key bias adds q_i . b_k to every score of row i: the softmax over the keys
    cancels it. A query bias does not cancel."""
    rng = np.random.default_rng(32)
    C, L, heads = 8, 9, 2
    w = _weights(rng, C)
    x = rng.normal(0, 1, (L, C))
    _, xp, s = _run(o, x, w, heads)
    w2 = dict(w, bqkv=w["bqkv"].copy())
    w2["bqkv"][C:2 * C] += rng.normal(0, 1.0, C)
    _, xp2, s2 = _run(o, x, w2, heads)
    assert np.allclose(xp2, xp, atol=1e-12, rtol=0)
    assert np.allclose(s2, s, atol=1e-12, rtol=0)
    w3 = dict(w, bqkv=w["bqkv"].copy())
    w3["bqkv"][:C] += rng.normal(0, 1.0, C)
    _, xp3, _ = _run(o, x, w3, heads)
    assert np.max(np.abs(xp3 - xp)) > 1e-4


def pin_attn_one_token(o):
    """L = 1: the softmax weight is 1, so SA(LN(x)) = (LN(x) W_v^T + b_v) W_o^T + b_o."""
    rng = np.random.default_rng(33)
    C = 8
    for heads in (1, 2, 4):
        w = _weights(rng, C)
        x = rng.normal(0, 1, (1, C))
        a, xp, s = _run(o, x, w, heads)
        u = rs_oracle.layer_norm(x, w["gamma"], w["beta"])
        v = u @ w["Wqkv"][2 * C:].T + w["bqkv"][2 * C:]
        want = v @ w["Wo"].T + w["bo"]
        assert np.allclose(a, want, atol=1e-12, rtol=0)
        assert np.allclose(xp, x + want, atol=1e-12, rtol=0)


def pin_attn_convex(o):
    """With W_o = I and b_o = 0 each output coordinate lies between the smallest
    and largest value of that coordinate over the tokens (softmax weights are
    non-negative and sum to 1), even with large scores."""
    rng = np.random.default_rng(34)
    C, L, heads = 8, 12, 4
    qkv = rng.normal(0, 6.0, (L, 3 * C))
    out = o.attention_core(qkv, heads)
    v = qkv[:, 2 * C:]
    assert np.all(out <= v.max(axis=0) + 1e-12) and np.all(out >= v.min(axis=0) - 1e-12)
    # a value column that is constant comes out as that constant
    qkv[:, 2 * C + 3] = 1.25
    assert np.allclose(o.attention_core(qkv, heads)[:, 3], 1.25, atol=1e-12, rtol=0)


def pin_attn_permutation(o):
    """Without position terms attention is permutation-equivariant over tokens:
    permuting the rows of x permutes x' and the shift."""
    rng = np.random.default_rng(35)
    C, L, heads = 8, 10, 2
    w = _weights(rng, C)
    x = rng.normal(0, 1, (L, C))
    perm = rng.permutation(L)
    _, xp, s = _run(o, x, w, heads)
    _, xq, sq = _run(o, x[perm], w, heads)
    assert np.allclose(xq, xp[perm], atol=1e-12, rtol=0)
    assert np.allclose(sq, s[perm], atol=1e-12, rtol=0)


def pin_attn_zero_sublayer(o):
    """W_o = 0, b_o = 0: SA(LN(x)) = 0, so x' = x and the shift D(0, x) is ||x||_2,
    ||x||_1, and 1 for the cosine distance (the floored denominator); pruning then
    keeps the tokens of largest norm."""
    rng = np.random.default_rng(36)
    C, L = 8, 6
    w = _weights(rng, C)
    w["Wo"] = np.zeros((C, C))
    w["bo"] = np.zeros(C)
    norms = np.array([0.5, 3.0, 1.0, 4.0, 2.0, 0.25])
    dirs = rng.normal(0, 1, (L, C))
    x = dirs / np.linalg.norm(dirs, axis=1, keepdims=True) * norms[:, None]
    for metric in ("l2", "l1", "cosine"):
        a, xp, s = _run(o, x, w, 2, metric)
        assert np.array_equal(xp, x)
        want = {"l2": norms, "l1": np.abs(x).sum(axis=1), "cosine": np.ones(L)}[metric]
        assert np.allclose(s, want, atol=1e-12, rtol=0), (metric, s)
    xk, kept, s, xp = o.attn_forward(x[None], w["Wqkv"], w["bqkv"], w["Wo"], w["bo"],
                                     w["gamma"], w["beta"], 2, keep_k=2)
    assert kept[0].tolist() == [0, 1, 3]       # CLS, then the norms 3.0 and 4.0
    assert np.array_equal(xk[0], x[[0, 1, 3]])
    _, kept_nc, _, _ = o.attn_forward(x[None], w["Wqkv"], w["bqkv"], w["Wo"], w["bo"],
                                      w["gamma"], w["beta"], 2, keep_k=3, cls=False)
    assert kept_nc[0].tolist() == [1, 3, 4]


def pin_attn_samples_independent(o):
    """Attention mixes tokens within a sample only: a batch gives what each sample
    gives alone."""
    rng = np.random.default_rng(37)
    C, L, heads = 8, 5, 2
    w = _weights(rng, C)
    x = rng.normal(0, 1, (3, L, C))
    args = (w["Wqkv"], w["bqkv"], w["Wo"], w["bo"], w["gamma"], w["beta"], heads)
    xp, s = o.attn_forward(x, *args)
    for b in range(3):
        xb, sb = o.attn_forward(x[b:b + 1], *args)
        assert np.array_equal(xb[0], xp[b]) and np.array_equal(sb[0], s[b])
    x2 = x.copy()
    x2[1] += rng.normal(0, 1, (L, C))
    xp2, _ = o.attn_forward(x2, *args)
    assert np.array_equal(xp2[0], xp[0]) and np.array_equal(xp2[2], xp[2])


ALL_ATTN_PINS = [pin_attn_hand_sublayer, pin_attn_hand_core, pin_attn_uniform_keys,
                 pin_attn_key_bias, pin_attn_one_token, pin_attn_convex, pin_attn_permutation,
                 pin_attn_zero_sublayer, pin_attn_samples_independent]
