"""The encoder oracle (layers of Eq. (5) + Eq. (6) with pruning between them) against
closed forms, and planted mistakes that those checks catch (CPU only)."""
import numpy as np
import pytest

from oracle import attn_oracle, encoder_oracle


def _layer(rng, C, H, mlp_zero=False, attn_zero=False):
    w = dict(Wqkv=rng.normal(0, 0.3, (3 * C, C)), bqkv=rng.normal(0, 0.1, 3 * C),
             Wo=rng.normal(0, 0.3, (C, C)), bo=rng.normal(0, 0.1, C),
             gamma1=1 + rng.normal(0, 0.1, C), beta1=rng.normal(0, 0.1, C),
             W1=rng.normal(0, 0.3, (H, C)), b1=rng.normal(0, 0.1, H),
             W2=rng.normal(0, 0.3, (C, H)), b2=rng.normal(0, 0.1, C),
             gamma2=1 + rng.normal(0, 0.1, C), beta2=rng.normal(0, 0.1, C))
    if attn_zero:
        w["Wo"], w["bo"] = np.zeros((C, C)), np.zeros(C)
    if mlp_zero:
        w["W2"], w["b2"] = np.zeros((C, H)), np.zeros(C)
    return w


def pin_schedule(e):
    """§4.2: 20% of the patch tokens pruned after layers 1, 4, 7 of a 12-layer DeiT:
    196 - 39 = 157, 157 - 31 = 126, 126 - 25 = 101 (39.2, 31.4, 25.2 rounded)."""
    assert e.deit_schedule() == [-1, 157, -1, -1, 126, -1, -1, 101, -1, -1, -1, -1]
    assert e.keep_after_pruning(10, 0.25) == 7          # 2.5 rounds to 3 (half up)
    assert e.keep_after_pruning(100) == 80


def pin_identity_layers(e):
    """W_o = 0, b_o = 0 and W2 = 0, b2 = 0 make every layer the identity, and the
    shift through the MLP is ||0 - x|| = ||x||: pruning keeps CLS and the patch
    tokens of largest norm, in index order, layer after layer."""
    rng = np.random.default_rng(41)
    C, H, L, B = 8, 16, 9, 2
    layers = [_layer(rng, C, H, mlp_zero=True, attn_zero=True) for _ in range(3)]
    norms = rng.permutation(np.arange(1, L + 1, dtype=np.float64))
    dirs = rng.normal(0, 1, (B, L, C))
    x = dirs / np.linalg.norm(dirs, axis=2, keepdims=True) * norms[None, :, None]
    out, kept = e.encoder_forward(x, layers, [-1, 5, 2], heads=2)
    for b in range(B):
        order = 1 + np.argsort(-norms[1:], kind="stable")   # patch tokens by norm
        k1 = np.sort(order[:5])
        k2 = np.sort(order[:2])
        assert kept[0][b].tolist() == [0] + k1.tolist()
        assert np.array_equal(out[b], x[b][[0] + k2.tolist()])


def pin_attention_layer(e):
    """With the MLP zeroed (W2 = 0, b2 = 0) a non-pruning layer is the attention
    sublayer alone: x + SA(LN(x))."""
    rng = np.random.default_rng(42)
    C, H, L = 8, 16, 6
    w = _layer(rng, C, H, mlp_zero=True)
    x = rng.normal(0, 1, (2, L, C))
    out, kept = e.encoder_forward(x, [w], [-1], heads=2)
    want, _ = attn_oracle.attn_forward(x, w["Wqkv"], w["bqkv"], w["Wo"], w["bo"], w["gamma1"],
                                       w["beta1"], 2)
    assert kept == [] and np.allclose(out, want, atol=1e-12, rtol=0)


PINS = [pin_schedule, pin_identity_layers, pin_attention_layer]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_encoder_pin(pin):
    pin(encoder_oracle)


def _forward_skipping_attention(x, layers, keep, heads, eps=1e-6):
    from oracle import rs_oracle
    cur = np.asarray(x, dtype=np.float64)
    kept_all = []
    for w, k in zip(layers, keep):
        mlp = dict(W1=w["W1"], b1=w["b1"], W2=w["W2"], b2=w["b2"], gamma=w["gamma2"],
                   beta=w["beta2"])
        if k >= 0:
            cur, kept, _, _ = rs_oracle.block_forward(cur, keep_k=k, **mlp)
            kept_all.append(kept)
        else:
            B, L, C = cur.shape
            cur = rs_oracle.sublayer(cur.reshape(B * L, C), **mlp)[1].reshape(B, L, C)
    return cur, kept_all


def _keep_truncating(patches, ratio=0.2):
    return patches - int(ratio * patches)   # 2.5 -> 2: keeps one token too many


def _schedule_ceiling(depth=12, L=197, layers=(1, 4, 7), ratio=0.2):
    import math
    keep = [-1] * depth
    p = L - 1
    for l in layers:
        p = p - math.ceil(ratio * p)        # 196 -> 156 -> 124 -> 99
        keep[l] = p
    return keep


MUTATIONS = {
    "attention_sublayer_skipped": ("encoder_forward", _forward_skipping_attention),
    "schedule_rounds_up": ("deit_schedule", _schedule_ceiling),
    "pruned_count_truncated": ("keep_after_pruning", _keep_truncating),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_encoder_pins_catch_mutation(name, monkeypatch):
    fn_name, bad = MUTATIONS[name]
    monkeypatch.setattr(encoder_oracle, fn_name, bad)
    caught = []
    for pin in PINS:
        try:
            pin(encoder_oracle)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches {name!r}"


def test_bench_schedule_matches_oracle():
    """bench.py's 12-layer timing uses the same pruning schedule as the oracle's reading
    of §4.2 (written separately there, since bench.py's timed path does not use the
    oracle)."""
    import bench
    assert bench.deit_keep_schedule(197) == encoder_oracle.deit_schedule()
    for L in (50, 101, 577):
        assert bench.deit_keep_schedule(L) == encoder_oracle.deit_schedule(L=L)
