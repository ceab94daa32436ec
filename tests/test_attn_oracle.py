"""The attention oracle against its pins, and planted mistakes that the pins must
catch (CPU only)."""
import numpy as np
import pytest

import oracle.attn_oracle as attn_oracle
from oracle import rs_oracle
from attn_pins import ALL_ATTN_PINS


@pytest.mark.parametrize("pin", ALL_ATTN_PINS, ids=lambda f: f.__name__)
def test_attn_pin(pin):
    pin(attn_oracle)


def _softmax_over_queries(S):
    e = np.exp(S - S.max(axis=-2, keepdims=True))
    return e / e.sum(axis=-2, keepdims=True)


def _softmax_unnormalised(S):
    return np.exp(S - S.max(axis=-1, keepdims=True))


def _core_with(scale_fn=None, v_from_k=False, merge_transposed=False, swap_qk=False):
    def core(qkv, heads):
        L, C3 = qkv.shape
        C = C3 // 3
        d = C // heads
        out = np.empty((L, C))
        for h in range(heads):
            q = qkv[:, h * d:(h + 1) * d]
            k = qkv[:, C + h * d:C + (h + 1) * d]
            v = qkv[:, (C if v_from_k else 2 * C) + h * d:(C if v_from_k else 2 * C) + (h + 1) * d]
            S = (k @ q.T if swap_qk else q @ k.T) * (scale_fn(d, C) if scale_fn else 1 / np.sqrt(d))
            o = attn_oracle.softmax_rows(S) @ v
            if merge_transposed:   # (L, d) blocks laid out as (d, L) and flattened per head
                out[:, h * d:(h + 1) * d] = o.T.reshape(-1)[: L * d].reshape(L, d)
            else:
                out[:, h * d:(h + 1) * d] = o
        return out
    return core


def _sublayer_shift_vs_output(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads, eps=rs_oracle.EPS,
                              metric="l2"):
    u = rs_oracle.layer_norm(x, gamma, beta, eps)
    a = rs_oracle.fc(attn_oracle.self_attention(u, Wqkv, bqkv, heads), Wo, bo)
    return a, x + a, rs_oracle.shift_score(a, x + a, metric)


def _sublayer_no_ln(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads, eps=rs_oracle.EPS, metric="l2"):
    a = rs_oracle.fc(attn_oracle.self_attention(x, Wqkv, bqkv, heads), Wo, bo)
    return a, x + a, rs_oracle.shift_score(a, x, metric)


def _sublayer_no_residual(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads, eps=rs_oracle.EPS,
                          metric="l2"):
    u = rs_oracle.layer_norm(x, gamma, beta, eps)
    a = rs_oracle.fc(attn_oracle.self_attention(u, Wqkv, bqkv, heads), Wo, bo)
    return a, a, rs_oracle.shift_score(a, x, metric)


def _sublayer_no_out_bias(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads, eps=rs_oracle.EPS,
                          metric="l2"):
    u = rs_oracle.layer_norm(x, gamma, beta, eps)
    a = attn_oracle.self_attention(u, Wqkv, bqkv, heads) @ Wo.T
    return a, x + a, rs_oracle.shift_score(a, x, metric)


def _forward_mixing_samples(x, Wqkv, bqkv, Wo, bo, gamma, beta, heads, keep_k=None,
                            eps=rs_oracle.EPS, metric="l2", cls=True):
    x = np.asarray(x, dtype=np.float64)
    B, L, C = x.shape
    _, xp, s = attn_oracle.attn_sublayer(x.reshape(B * L, C), Wqkv, bqkv, Wo, bo, gamma, beta,
                                         heads, eps, metric)
    xp, s = xp.reshape(B, L, C), s.reshape(B, L)
    if keep_k is None:
        return xp, s
    kept = np.stack([rs_oracle.select_topk(s[b], keep_k, cls) for b in range(B)])
    return np.stack([xp[b][kept[b]] for b in range(B)]), kept, s, xp


MUTATIONS = {
    "softmax_over_queries": ("softmax_rows", _softmax_over_queries),
    "softmax_unnormalised": ("softmax_rows", _softmax_unnormalised),
    "scale_one_over_d": ("attention_core", _core_with(scale_fn=lambda d, C: 1.0 / d)),
    "no_scale": ("attention_core", _core_with(scale_fn=lambda d, C: 1.0)),
    "scale_sqrt_C_per_head": ("attention_core", _core_with(scale_fn=lambda d, C: 1 / np.sqrt(C))),
    "v_from_key_slice": ("attention_core", _core_with(v_from_k=True)),
    "heads_merged_transposed": ("attention_core", _core_with(merge_transposed=True)),
    "scores_transposed": ("attention_core", _core_with(swap_qk=True)),
    "shift_against_output": ("attn_sublayer", _sublayer_shift_vs_output),
    "no_layernorm": ("attn_sublayer", _sublayer_no_ln),
    "no_residual": ("attn_sublayer", _sublayer_no_residual),
    "no_output_bias": ("attn_sublayer", _sublayer_no_out_bias),
    "samples_mixed": ("attn_forward", _forward_mixing_samples),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_attn_pins_catch_mutation(name, monkeypatch):
    fn_name, bad = MUTATIONS[name]
    monkeypatch.setattr(attn_oracle, fn_name, bad)
    caught = []
    for pin in ALL_ATTN_PINS:
        try:
            pin(attn_oracle)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"
