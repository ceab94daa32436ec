"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each ``pin_*`` takes the oracle *module* and raises AssertionError when the
oracle disagrees with the fact. Calls go through the module's attributes, so a
test can plant a mistake in one oracle function (monkeypatch) and check that at
least one pin catches it.

Sources of truth used here:
* a standard normal CDF table (GELU(z) = z * Phi(z));
* a hand-worked 4-token case with identity weights (tests/golden/);
* closed forms of Eq. (6) for degenerate weights (W2 = 0, W1 = 0);
* explicit index-by-index loops for LayerNorm and the two contractions;
* exhaustive subset search for the kept set;
* invariants: permutation equivariance (the MLP acts on each token alone,
  §3.3), CLS always kept, LayerNorm output moments.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _identity_weights(C):
    eye = np.eye(C)
    z = np.zeros(C)
    return dict(W1=eye, b1=z, W2=eye, b2=z, gamma=np.ones(C), beta=z)


def _rng_weights(rng, C, H):
    return dict(
        W1=rng.normal(0, 0.3, (H, C)), b1=rng.normal(0, 0.1, H),
        W2=rng.normal(0, 0.3, (C, H)), b2=rng.normal(0, 0.1, C),
        gamma=1 + rng.normal(0, 0.2, C), beta=rng.normal(0, 0.1, C),
    )


def pin_gelu_table(o):
    """GELU(z) = z Phi(z) and GELU(-z) = -z (1 - Phi(z)) at tabulated points."""
    tab = _golden("normal_cdf_table.json")["phi"]
    for zs, phi in tab.items():
        z = float(zs)
        got = o.gelu(np.array([z, -z, 0.0]))
        assert abs(got[0] - z * phi) < 1e-12, (z, got[0], z * phi)
        assert abs(got[1] - (-z * (1.0 - phi))) < 1e-12, (z, got[1])
        assert got[2] == 0.0


def pin_hand_example(o):
    """The 4-token identity-weight case: scores, outputs and kept sets."""
    g = _golden("hand_example_4tok.json")
    phi1 = _golden("normal_cdf_table.json")["phi"]["1.0"]
    phim1 = 1.0 - phi1
    x = np.array(g["x"], dtype=np.float64)
    w = _identity_weights(4)
    h, y, s = o.sublayer(x, eps=0.0, **w)
    h_row = np.array([phi1, -phim1, phi1, -phim1])
    for t in range(4):
        assert np.allclose(h[t], h_row, rtol=0, atol=1e-12), (t, h[t])
        assert np.allclose(y[t], x[t] + h_row, rtol=0, atol=1e-12)
    s_exp = [
        math.sqrt(2 * ((2 - phi1) ** 2 + phim1 ** 2)),
        math.sqrt(2 * (phim1 ** 2 + phi1 ** 2)),
        math.sqrt(2 * ((3 - phi1) ** 2 + (1 + phim1) ** 2)),
        math.sqrt(2 * (phim1 ** 2 + phi1 ** 2)),
    ]
    assert np.allclose(s, s_exp, rtol=0, atol=1e-12), (s, s_exp)
    for k, kept in g["kept_idx"].items():
        got = o.select_topk(s, int(k))
        assert list(got) == kept, (k, list(got), kept)
        yk, kidx, sc, _ = o.block_forward(x[None], keep_k=int(k), eps=0.0, **w)
        assert list(kidx[0]) == kept
        assert np.array_equal(yk[0], (x + h_row)[kept])
    # the constant row: variance 0, u = beta = 0 exactly for any eps > 0
    cr = g["constant_row"]
    xc = np.array([[2.0, 2.0, 2.0, 2.0]])
    h, y, s = o.sublayer(xc, eps=1e-6, **w)
    assert np.array_equal(h[0], np.array(cr["h"], dtype=float)), h
    assert s[0] == cr["s"] and np.array_equal(y[0], np.array(cr["y"], dtype=float))


def pin_zero_shift(o):
    """W2 = 0 gives h = b2 for every token, so a row equal to b2 has s = 0 (Eq. (4))."""
    rng = np.random.default_rng(11)
    C, H, L = 6, 10, 5
    w = _rng_weights(rng, C, H)
    w["W2"] = np.zeros((C, H))
    x = rng.normal(0, 1, (L, C))
    x[2] = w["b2"]
    h, y, s = o.sublayer(x, **w)
    assert np.allclose(h, np.broadcast_to(w["b2"], h.shape), rtol=0, atol=1e-15)
    assert s[2] == 0.0, s
    for t in range(L):
        assert abs(s[t] - math.sqrt(sum((w["b2"][c] - x[t, c]) ** 2 for c in range(C)))) < 1e-12
    assert np.allclose(y, x + w["b2"], rtol=0, atol=1e-15)


def pin_first_layer_zero(o):
    """W1 = 0 gives the constant h = W2 GELU(b1) + b2 for every token."""
    rng = np.random.default_rng(12)
    C, H, L = 5, 7, 4
    w = _rng_weights(rng, C, H)
    w["W1"] = np.zeros((H, C))
    x = rng.normal(0, 1, (L, C))
    a = [o.gelu(np.array([w["b1"][j]]))[0] for j in range(H)]
    h_exp = [sum(w["W2"][c][j] * a[j] for j in range(H)) + w["b2"][c] for c in range(C)]
    h, _, _ = o.sublayer(x, **w)
    for t in range(L):
        assert np.allclose(h[t], h_exp, rtol=0, atol=1e-12)


def pin_loops(o):
    """LayerNorm, fc1, fc2, the residual and the score, index by index."""
    # the square case first: a transposed weight then fails an assertion rather than
    # a shape check
    for seed, (C, H, L) in ((14, (4, 4, 3)), (13, (3, 5, 4))):
        _loops_case(o, np.random.default_rng(seed), C, H, L)


def _loops_case(o, rng, C, H, L):
    w = _rng_weights(rng, C, H)
    x = rng.normal(0, 1, (L, C)) * 2 + 0.5
    h, y, s = o.sublayer(x, **w)
    for t in range(L):
        mu = sum(x[t]) / C
        var = sum((x[t][c] - mu) ** 2 for c in range(C)) / C
        u = [(x[t][c] - mu) / math.sqrt(var + 1e-6) * w["gamma"][c] + w["beta"][c] for c in range(C)]
        z = [sum(w["W1"][j][c] * u[c] for c in range(C)) + w["b1"][j] for j in range(H)]
        a = [o.gelu(np.array([zj]))[0] for zj in z]
        hh = [sum(w["W2"][c][j] * a[j] for j in range(H)) + w["b2"][c] for c in range(C)]
        ss = math.sqrt(sum((hh[c] - x[t][c]) ** 2 for c in range(C)))
        assert np.allclose(h[t], hh, rtol=0, atol=1e-12), (t, h[t], hh)
        assert np.allclose(y[t], [hh[c] + x[t][c] for c in range(C)], rtol=0, atol=1e-12)
        assert abs(s[t] - ss) < 1e-12


def pin_ln_moments(o):
    """With gamma = 1, beta = 0, eps = 0 each LN row has mean 0 and mean square 1."""
    rng = np.random.default_rng(14)
    x = rng.normal(3.0, 2.0, (16, 64))
    u = o.layer_norm(x, np.ones(64), np.zeros(64), eps=0.0)
    assert np.abs(u.mean(axis=1)).max() < 1e-12
    assert np.abs((u ** 2).mean(axis=1) - 1.0).max() < 1e-12


def _unique_topk_by_dominance(s, k, first=1):
    """All k-subsets S of first..L-1 such that every kept token beats every dropped one
    (larger s, or equal s and lower index). Exactly one exists."""
    L = len(s)
    pats = range(first, L)
    out = []
    for S in itertools.combinations(pats, k):
        Sset = set(S)
        ok = all(
            (s[i] > s[j]) or (s[i] == s[j] and i < j)
            for i in Sset for j in pats if j not in Sset
        )
        if ok:
            out.append(S)
    return out


def pin_topk_exhaustive(o):
    """Kept set = the unique dominance-closed k-subset, for every k, with ties."""
    rng = np.random.default_rng(15)
    for L in (2, 3, 6, 9, 11):
        for trial in range(3):
            s = rng.integers(0, 4, L).astype(np.float64) * 0.5  # many exact ties
            if trial == 2:
                s = rng.random(L)
            for k in range(0, L):
                sols = _unique_topk_by_dominance(s, k)
                assert len(sols) == 1
                got = o.select_topk(s, k)
                assert got[0] == 0 and len(got) == 1 + k
                assert list(got[1:]) == list(sols[0]), (L, k, s, got, sols)


def pin_permutation(o):
    """Permuting patch rows permutes the scores bit for bit and maps the kept set."""
    rng = np.random.default_rng(16)
    C, H, L, k = 8, 16, 12, 5
    w = _rng_weights(rng, C, H)
    x = rng.normal(0, 1, (1, L, C))
    perm = np.concatenate([[0], 1 + rng.permutation(L - 1)])
    yk, kept, s, y = o.block_forward(x, keep_k=k, **w)
    yk2, kept2, s2, y2 = o.block_forward(x[:, perm], keep_k=k, **w)
    assert np.array_equal(s2[0], s[0][perm])
    assert len(set(s[0][1:])) == L - 1  # distinct scores: the tie rule plays no part
    inv = np.argsort(perm)
    assert sorted(perm[kept2[0]]) == sorted(kept[0])
    assert np.array_equal(y2[0], y[0][perm])
    assert kept2[0][0] == 0 and np.all(np.diff(kept2[0]) > 0)
    assert np.array_equal(yk2[0], y2[0][kept2[0]])
    assert inv[0] == 0


def pin_cls_kept(o):
    """CLS is kept first even when its score is the lowest (here exactly 0)."""
    rng = np.random.default_rng(17)
    C, H, L = 8, 16, 10
    w = _rng_weights(rng, C, H)
    w["b1"] = np.zeros(H)
    w["b2"] = np.zeros(C)
    w["beta"] = np.zeros(C)
    x = rng.normal(0, 1, (1, L, C))
    x[0, 0] = 0.0
    for k in range(0, L):
        yk, kept, s, y = o.block_forward(x, keep_k=k, **w)
        assert s[0, 0] == 0.0 and s[0, 1:].min() > 0
        assert kept[0][0] == 0 and 0 not in list(kept[0][1:])
        assert len(kept[0]) == 1 + k


def pin_metrics_hand_example(o):
    """L1 and cosine distances (§3.3 "Distance metrics" (ii), (iii)) on the 4-token
    identity-weight case, by hand from Phi(1): every row has h = [P, -Q, P, -Q] with
    P = Phi(1), Q = Phi(-1) = 1 - P, so h - x and h.x follow row by row. The kept sets
    differ by metric (cosine ranks t1, t3 above t2), and without a CLS token t0 competes."""
    g = _golden("hand_example_4tok.json")
    P = _golden("normal_cdf_table.json")["phi"]["1.0"]
    Q = 1.0 - P
    x = np.array(g["x"], dtype=np.float64)
    w = _identity_weights(4)
    nh = math.sqrt(2 * (P * P + Q * Q))
    l1 = [2 + 4 * Q, 2.0, 6 + 4 * Q, 2.0]
    cos = [1 - 4 * P / (math.sqrt(8) * nh), 1 - 1 / nh,
           1 - (6 * P - 2 * Q) / (math.sqrt(20) * nh), 1 - 1 / nh]
    _, _, s1 = o.sublayer(x, eps=0.0, metric="l1", **w)
    assert np.allclose(s1, l1, rtol=0, atol=1e-12), (s1, l1)
    _, _, sc = o.sublayer(x, eps=0.0, metric="cosine", **w)
    assert np.allclose(sc, cos, rtol=0, atol=1e-12), (sc, cos)
    expect = {
        ("l1", True): {0: [0], 1: [0, 2], 2: [0, 1, 2], 3: [0, 1, 2, 3]},
        ("cosine", True): {0: [0], 1: [0, 1], 2: [0, 1, 3], 3: [0, 1, 2, 3]},
        # no CLS: L2 scores 1.65, 1.21, 3.46, 1.21 rank t2, t0, then the tied t1, t3
        ("l2", False): {0: [], 1: [2], 2: [0, 2], 3: [0, 1, 2], 4: [0, 1, 2, 3]},
        ("cosine", False): {0: [], 1: [1], 2: [1, 3], 3: [1, 2, 3], 4: [0, 1, 2, 3]},
    }
    for (metric, cls), kept_by_k in expect.items():
        for k, kept in kept_by_k.items():
            yk, kidx, sc_, _ = o.block_forward(x[None], keep_k=k, eps=0.0, metric=metric,
                                               cls=cls, **w)
            assert list(kidx[0]) == kept, (metric, cls, k, list(kidx[0]), kept)
            assert yk.shape == (1, len(kept), 4)


def pin_metric_invariants(o):
    """Norm inequalities between L1 and L2, the range of the cosine distance, its
    indifference to the length of h, and parallel / antiparallel / orthogonal cases."""
    rng = np.random.default_rng(19)
    C = 16
    h = rng.normal(0, 1, (6, C))
    x = rng.normal(0, 1, (6, C))
    l2, l1, cs = (o.shift_score(h, x, m) for m in ("l2", "l1", "cosine"))
    assert np.all(l1 >= l2 - 1e-12) and np.all(l1 <= math.sqrt(C) * l2 + 1e-12)
    assert np.all(cs >= 0) and np.all(cs <= 2)
    # scaling h by 2 is exact in binary floating point: the cosine distance is unchanged
    # bit for bit, while L1 and L2 are not
    assert np.array_equal(o.shift_score(2 * h, x, "cosine"), cs)
    assert not np.allclose(o.shift_score(2 * h, x, "l2"), l2)
    v = x[:1]
    assert abs(o.shift_score(v, v, "cosine")[0]) < 1e-15
    assert abs(o.shift_score(-v, v, "cosine")[0] - 2.0) < 1e-15
    e = np.eye(C)
    assert o.shift_score(e[:1], e[1:2], "cosine")[0] == 1.0
    d = np.zeros((1, C))
    d[0, 3] = -2.5
    assert o.shift_score(x[:1] + d, x[:1], "l1")[0] == 2.5
    assert o.shift_score(x[:1] + d, x[:1], "l2")[0] == 2.5


def pin_topk_no_cls_exhaustive(o):
    """Without a CLS token: kept set = the unique dominance-closed k-subset of all L
    tokens, for every k, with ties."""
    rng = np.random.default_rng(20)
    for L in (1, 2, 5, 8, 10):
        for trial in range(3):
            s = rng.integers(0, 4, L).astype(np.float64) * 0.5
            if trial == 2:
                s = rng.random(L)
            for k in range(0, L + 1):
                sols = _unique_topk_by_dominance(s, k, first=0)
                assert len(sols) == 1
                got = o.select_topk(s, k, cls=False)
                assert list(got) == list(sols[0]), (L, k, s, got, sols)


def pin_permutation_no_cls(o):
    """Without a CLS token, permuting all rows (t0 included) permutes the scores and maps
    the kept set."""
    rng = np.random.default_rng(21)
    C, H, L, k = 8, 16, 11, 4
    w = _rng_weights(rng, C, H)
    x = rng.normal(0, 1, (1, L, C))
    perm = rng.permutation(L)
    for metric in ("l2", "cosine"):
        yk, kept, s, y = o.block_forward(x, keep_k=k, metric=metric, cls=False, **w)
        yk2, kept2, s2, y2 = o.block_forward(x[:, perm], keep_k=k, metric=metric, cls=False, **w)
        assert np.array_equal(s2[0], s[0][perm])
        assert len(set(s[0])) == L
        assert sorted(perm[kept2[0]]) == sorted(kept[0]) and len(kept[0]) == k
        assert np.all(np.diff(kept2[0]) > 0)
        assert np.array_equal(yk2[0], y2[0][kept2[0]])


def pin_block_shift(o):
    """The whole-block shift D(y, x_in) (§3.3 case (iii)). With W2 = 0, b2 = 0 the MLP
    adds nothing, y = x', and the shift is D(x', x_in): built here as x_in = x' - delta
    with rows of known size, so s_l2 = ||delta||, s_l1 = sum |delta| and pruning keeps
    the largest deltas. With x_in = x' and b2 = c the shift is ||h|| = ||c|| for every
    token: all scores tie and the lowest indices are kept."""
    rng = np.random.default_rng(22)
    C, H, L = 8, 16, 7
    w = _rng_weights(rng, C, H)
    w["W2"] = np.zeros((C, H))
    w["b2"] = np.zeros(C)
    xp = rng.normal(0, 1, (1, L, C))
    sizes = np.array([0.5, 2.0, 0.25, 3.0, 1.0, 4.0, 1.5])
    d = rng.normal(0, 1, (L, C))
    delta = d / np.linalg.norm(d, axis=1, keepdims=True) * sizes[:, None]
    x_in = xp - delta[None]
    for metric in ("l2", "l1"):
        yk, kept, s, y = o.block_shift_forward(x_in, xp, keep_k=3, metric=metric, **w)
        assert np.array_equal(y, xp)
        want = sizes if metric == "l2" else np.abs(delta).sum(axis=1)
        assert np.allclose(s[0], want, atol=1e-12, rtol=0), (metric, s)
    _, kept, _, _ = o.block_shift_forward(x_in, xp, keep_k=3, **w)
    assert kept[0].tolist() == [0, 1, 3, 5]          # CLS, then sizes 2.0, 3.0, 4.0
    c = rng.normal(0, 1, C)
    w["b2"] = c
    _, kept, s, y = o.block_shift_forward(xp, xp, keep_k=3, **w)
    assert np.allclose(s[0], np.linalg.norm(c), atol=1e-12, rtol=0)
    assert kept[0].tolist() == [0, 1, 2, 3]


def pin_gather(o):
    """The kept rows of y, in kept order."""
    rng = np.random.default_rng(18)
    y = rng.normal(0, 1, (7, 3))
    kept = np.array([0, 2, 5, 6])
    assert np.array_equal(o.gather(y, kept), np.stack([y[0], y[2], y[5], y[6]]))


ALL_PINS = [
    pin_gelu_table,
    pin_block_shift,
    pin_metrics_hand_example,
    pin_metric_invariants,
    pin_topk_no_cls_exhaustive,
    pin_permutation_no_cls,
    pin_hand_example,
    pin_zero_shift,
    pin_first_layer_zero,
    pin_loops,
    pin_ln_moments,
    pin_topk_exhaustive,
    pin_permutation,
    pin_cls_kept,
    pin_gather,
]
