"""The CPU model of the kernels' rounding points (tests/kernel_model.py), on the CPU.

1. With every rounding point switched off the model is the oracle (float64
   agreement), so it differs from the oracle only where it rounds.
2. On the attention sublayer's ill-conditioned inputs (weights of std 0.05 at
   C = 1024, std 0.05 with a small residual at C = 768, std 0.1 with peaked
   softmax rows) the rounding alone -- no kernel involved -- leaves the parity
   tolerance against the oracle. This is why those inputs are compared with the
   model rather than with the oracle on the GPU (tests/test_attn_gpu.py).
3. On the well-conditioned inputs the model stays inside the tolerance.
4. The fp32 score finalisation on exactly representable partials, with two
   planted mistakes caught.
"""
import numpy as np
import pytest

import kernel_model as km
import parity
from attn_cases import CONDITIONED, ILL_CONDITIONED, attn_case, case_id, w64
from oracle import attn_oracle, rs_oracle


@pytest.mark.parametrize("case", CONDITIONED[:2] + ILL_CONDITIONED[2:4])
def test_model_without_rounding_is_the_oracle(case):
    x, w = attn_case(*case)
    x64, W = parity.f64(x), w64(w)
    heads = x.shape[2] // 64
    ref, _ = attn_oracle.attn_forward(x64, heads=heads, **W)
    got = km.attn_sublayer_bf16(x64, heads=heads, rounding=False, **W)
    assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
    # the pieces: the folded projection is LN then the linear map; the blocked core
    # with a lagging reference maximum is the softmax attention
    u = rs_oracle.layer_norm(x64[0], W["gamma"], W["beta"])
    z = km.folded_projection(x64[0], W["Wqkv"], W["bqkv"], W["gamma"], W["beta"], rounding=False)
    zr = rs_oracle.fc(u, W["Wqkv"], W["bqkv"])
    assert np.abs(z - zr).max() <= 1e-12 * np.abs(zr).max()
    qkv = zr * 4.0  # sharper rows: the reference maximum moves between key blocks
    core = km.attention_core_bf16(qkv, heads, rounding=False)
    core_r = attn_oracle.attention_core(qkv, heads)
    assert np.abs(core - core_r).max() <= 1e-12 * np.abs(core_r).max()


@pytest.mark.parametrize("case", ILL_CONDITIONED, ids=case_id)
def test_rounding_alone_leaves_the_tolerance(case):
    """The kernels' bf16 rounding points, modelled on the CPU, already put elements of
    x' outside 2e-2 max(1, |ref|) of the fp64 oracle on these inputs."""
    x, w = attn_case(*case)
    x64, W = parity.f64(x), w64(w)
    heads = x.shape[2] // 64
    ref, _ = attn_oracle.attn_forward(x64, heads=heads, **W)
    model = km.attn_sublayer_bf16(x64, heads=heads, **W)
    with pytest.raises(AssertionError, match="outside"):
        parity.check_y(model, ref, "model")


@pytest.mark.parametrize("case", CONDITIONED, ids=case_id)
def test_model_within_tolerance_when_conditioned(case):
    x, w = attn_case(*case)
    x64, W = parity.f64(x), w64(w)
    heads = x.shape[2] // 64
    ref, _ = attn_oracle.attn_forward(x64, heads=heads, **W)
    parity.check_y(km.attn_sublayer_bf16(x64, heads=heads, **W), ref, "model")


def test_fold_rounding_is_what_the_qkv_only_model_missed():
    """On the peaked std 0.1 case, rounding only the stored QKV projection (and not
    the folded weights bf16(W gamma)) falls short of the full model by more than
    the tolerance on some elements: the folded weights' rounding is a first-order
    term of the error, comparable to the projection's."""
    x, w = attn_case(2, 138, 384, 0.1, 1.0, 1)
    x64, W = parity.f64(x), w64(w)
    heads = 6
    full = km.attn_sublayer_bf16(x64, heads=heads, **W)
    b = 0
    u = rs_oracle.layer_norm(x64[b], W["gamma"], W["beta"])
    qkv = km.bf16(rs_oracle.fc(u, W["Wqkv"], W["bqkv"]))
    qkv_only = x64[b] + rs_oracle.fc(attn_oracle.attention_core(qkv, heads), W["Wo"], W["bo"])
    d = np.abs(qkv_only - full[b])
    assert (d > 2e-2 * np.maximum(1.0, np.abs(full[b]))).any()


# ----------------------------------------------------------------------------- fp32 scores
def check_finalize(f):
    """fp32 score finalisation of each metric on exactly representable cases, and
    against its fp64 definition on random partials within fp32 rounding."""
    assert f(np.array([[9.0, 16.0]]), 1, 1, "l2")[0, 0] == 5.0
    assert f(np.array([[0.5, 0.25, 1.0]]), 1, 1, "l1")[0, 0] == 1.75
    tri = np.array([[4.0, 4.0, 4.0],      # parallel: 1 - 4 / (2 * 2) = 0
                    [0.0, 4.0, 9.0],      # orthogonal: 1
                    [-6.0, 4.0, 9.0],     # antiparallel: 1 + 6 / 6 = 2
                    [4.0, 2.0, 8.0],      # |h.x| above ||h|| ||x||: floored at 0
                    [0.0, 0.0, 9.0]])     # h = 0: 1 - 0 / 1e-8 = 1
    got = f(tri, 1, 5, "cosine")[0]
    assert list(got) == [0.0, 1.0, 2.0, 0.0, 1.0], got
    # two column groups: the triples are summed component-wise first
    two = np.array([[1.0, 1.0, 2.0, 1.0, 3.0, 2.0]])  # HX = 2, HH = 4, XX = 4
    assert f(two, 1, 1, "cosine")[0, 0] == 0.5
    rng = np.random.default_rng(22)
    p = rng.random((40, 6)).astype(np.float32)
    p64 = p.astype(np.float64)
    assert np.allclose(f(p, 1, 40, "l2")[0], np.sqrt(p64.sum(1)), rtol=1e-6)
    assert np.allclose(f(p, 1, 40, "l1")[0], p64.sum(1), rtol=1e-6)
    hx, hh, xx = p64[:, 0::3].sum(1), p64[:, 1::3].sum(1), p64[:, 2::3].sum(1)
    ref = np.maximum(1 - hx / np.sqrt(hh * xx), 0)
    assert np.allclose(f(p, 1, 40, "cosine")[0], ref, rtol=0, atol=1e-6)


def test_finalize_scores_f32():
    check_finalize(km.finalize_scores_f32)


def _cos_not_floored(partials, B, L, metric="l2"):
    if metric != "cosine":
        return km.finalize_scores_f32(partials, B, L, metric)
    p = np.asarray(partials, dtype=np.float32).reshape(B * L, -1)
    hx, hh, xx = (p[:, i::3].sum(1, dtype=np.float32) for i in range(3))
    return (1 - hx / (np.sqrt(hh) * np.sqrt(xx) + np.float32(1e-8))).reshape(B, L)


def _l1_takes_sqrt(partials, B, L, metric="l2"):
    return km.finalize_scores_f32(partials, B, L, "l2" if metric == "l1" else metric)


@pytest.mark.parametrize("bad", [_cos_not_floored, _l1_takes_sqrt])
def test_finalize_mistakes_caught(bad):
    with pytest.raises(AssertionError):
        check_finalize(bad)
