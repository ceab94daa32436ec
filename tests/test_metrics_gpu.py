"""The paper's other shift distances (L1, cosine; §3.3 "Distance metrics") and the
no-CLS mode (all L tokens ranked, as for UMT's patch-only sequences) on the CUDA path,
against the fp64 oracle through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import kernel_model
import oracle
import parity
from workloads import WORKLOADS, make_inputs, random_block, random_partials

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")
METRICS = ["l2", "l1", "cosine"]


def _rs():
    import free_vit_token_b200 as rs  # deferred: collection must not need a GPU
    return rs


def _partials(B, L, metric, seed, ties):
    """Select-kernel inputs: non-negative sums (L2, L1), or per-group triples
    (h.x signed, h.h and x.x non-negative) for the cosine distance."""
    P = 6
    p = random_partials(B, L, P, seed=seed, ties=ties)
    if metric == "cosine":
        p[:, 0::3] -= 1.0
    return p.contiguous()


@pytest.mark.parametrize("metric", METRICS)
@pytest.mark.parametrize("cls", [True, False])
@pytest.mark.parametrize("L", [1, 2, 197, 256, 257, 1098, 1569])
@pytest.mark.parametrize("ties", [False, True])
def test_select_metrics_bitexact(metric, cls, L, ties):
    """fp32 finalisation of each distance and the top-k with or without CLS: scores and
    kept lists bit-exact against the oracle's selection of the same fp32 keys."""
    rs = _rs()
    B = 3
    parts = _partials(B, L, metric, seed=L + 11 * ties + 5 * cls, ties=ties)
    s_ref = kernel_model.finalize_scores_f32(parts.numpy(), B, L, metric)
    n = L - (1 if cls else 0)  # ranked tokens
    ks = sorted({0, min(1, n), n // 2, max(n - 1, 0), n})
    pd = parts.to(dev)
    y = torch.randn(B, L, 64, generator=torch.Generator().manual_seed(L)).to(torch.bfloat16)
    yd = y.to(dev)
    for k in ks:
        scores, kept = rs.rs_select_topk(pd, B, L, k, distance=metric, cls=cls)
        sg_scores, sg_kept, y_kept = rs.rs_select_gather(pd, yd, k, distance=metric, cls=cls)
        torch.cuda.synchronize()
        assert np.array_equal(scores.cpu().numpy(), s_ref), "fp32 scores differ"
        assert torch.equal(sg_scores, scores) and torch.equal(sg_kept, kept)
        for b in range(B):
            ref = oracle.select_topk(s_ref[b].astype(np.float64), k, cls)
            got = kept[b].cpu().numpy().tolist()
            assert got == ref.tolist(), (metric, cls, L, k, b)
            assert torch.equal(y_kept[b].cpu(), y[b][ref])


@pytest.mark.parametrize("metric", ["l1", "cosine"])
@pytest.mark.parametrize("M,C,H", [(394, 192, 768), (130, 384, 1536), (300, 1024, 4096)])
def test_fc2_metric_partials(metric, M, C, H):
    """fc2's partials for L1 and cosine (single CTAs and CTA pairs), finalised in fp32,
    against the fp64 distance of the same h and x'; y unchanged."""
    rs = _rs()
    inp = random_block(1, M, C, H, seed=M + C, fg_rows=M // 4)
    x = inp.x.reshape(M, C)
    w = inp.weights[0]
    g = torch.Generator().manual_seed(M * 5 + 3)
    a = (torch.randn(M, H, generator=g) * 0.3).to(torch.bfloat16)
    y, parts = rs.rs_fc2_residual_shift(a.to(dev), x.to(dev), w.W2.to(dev), w.b2.to(dev),
                                        distance=metric)
    torch.cuda.synchronize()
    assert parts.shape == (M, rs.rs_num_partials(C, metric))
    w64 = parity.weights64(w)
    x64 = parity.f64(x)
    h = oracle.fc(parity.f64(a), w64["W2"], w64["b2"])
    parity.check_y(parity.f64(y), h + x64, "y")
    s_gpu = kernel_model.finalize_scores_f32(parts.cpu().numpy(), 1, M, metric)[0].astype(np.float64)
    parity.check_scores(s_gpu, oracle.shift_score(h, x64, metric))
    assert rs.rs_get_last_device_error() == 0


@pytest.mark.parametrize("metric", METRICS)
@pytest.mark.parametrize("cls", [True, False])
@pytest.mark.parametrize("B,L,C,H", [(2, 197, 192, 768), (2, 600, 128, 256), (3, 50, 128, 256)])
def test_block_metrics(metric, cls, B, L, C, H):
    """rs_block_forward with each distance, with and without CLS (rank path for L <= 256,
    radix path above), every keep_k edge, against the oracle."""
    rs = _rs()
    inp = random_block(B, L, C, H, seed=B * L + C, fg_rows=L // 3)
    W = [t.to(dev) for t in (inp.weights[0].W1, inp.weights[0].b1, inp.weights[0].W2,
                             inp.weights[0].b2, inp.weights[0].gamma, inp.weights[0].beta)]
    n = L - (1 if cls else 0)
    for k in sorted({0, 1, n // 2, n}):
        gpu = rs.rs_block_forward(inp.x.to(dev), *W, k, distance=metric, cls=cls)
        torch.cuda.synchronize()
        ref = parity.oracle_block(inp.x, inp.weights[0], k, metric, cls)
        parity.check_block(gpu, ref, k, cls=cls)
    assert rs.rs_get_last_device_error() == 0


@pytest.mark.parametrize("name,metric,cls", [("deit_s", "l1", True), ("deit_s", "cosine", True),
                                             ("umt_b", "l2", False)])
def test_config_metrics(name, metric, cls):
    """Full-batch configs with another distance, or UMT-B without its CLS token (the
    paper's UMT has none); a seeded subset of samples checked."""
    rs = _rs()
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0)
    k = wl.keep_k[0]
    w = inp.weights[0]
    W = [t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]
    gpu = rs.rs_block_forward(inp.x.to(dev), *W, k, distance=metric, cls=cls)
    torch.cuda.synchronize()
    samples = [0, wl.B // 2, wl.B - 1] if name.startswith("umt") else [0, 7, 100, wl.B - 1]
    ref = parity.oracle_block(inp.x[samples], w, k, metric, cls)
    res = parity.check_block(gpu, ref, k, samples, cls=cls)
    print(name, metric, cls, res)
    assert rs.rs_get_last_device_error() == 0
