"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

import kernel_model
import oracle
import parity
from workloads import WORKLOADS, make_inputs, random_block, random_partials

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")


def _rs():
    import free_vit_token_b200 as rs  # deferred: collection must not need a GPU
    return rs


def _to_dev(w):
    return [t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]


def _device_ok():
    rs = _rs()
    assert rs.rs_get_last_device_error() == 0


# --------------------------------------------------------------------------- select
@pytest.mark.parametrize("L", [1, 2, 3, 197, 256, 257, 1098, 1569, 4100])
@pytest.mark.parametrize("ties", [False, True])
def test_select_bitexact(L, ties):
    """fp32 score finalisation and top-k: bit-exact against the oracle's selection of
    the same fp32 keys (both sides finalise in fp32, sum left to right)."""
    rs = _rs()
    B, P = 3, 6
    parts = random_partials(B, L, P, seed=L + 7 * ties, ties=ties)
    s_ref = kernel_model.finalize_scores_f32(parts.numpy(), B, L)
    ks = sorted({0, min(1, L - 1), (L - 1) // 2, max(L - 2, 0), L - 1})
    pd = parts.to(dev)
    for k in ks:
        scores, kept = rs.rs_select_topk(pd, B, L, k)
        torch.cuda.synchronize()
        assert np.array_equal(scores.cpu().numpy(), s_ref), "fp32 scores differ"
        for b in range(B):
            ref = oracle.select_topk(s_ref[b].astype(np.float64), k)
            assert kept[b].cpu().numpy().tolist() == ref.tolist(), (L, k, b)


def test_select_cls_lowest_and_empty_batch():
    rs = _rs()
    B, L, P = 2, 50, 1
    parts = random_partials(B, L, P, seed=3) + 1.0
    parts[0] = 0.0  # CLS of sample 0 has score 0
    scores, kept = rs.rs_select_topk(parts.to(dev), B, L, 10)
    assert kept[0, 0].item() == 0 and 0 not in kept[0, 1:].tolist()
    e_s, e_k = rs.rs_select_topk(torch.empty(0, 1, device=dev), 0, L, 3)
    assert e_k.numel() == 0


# --------------------------------------------------------------------------- gather
@pytest.mark.parametrize("C", [64, 192, 384, 768, 1024, 2048])
def test_gather_exact(C):
    rs = _rs()
    g = torch.Generator().manual_seed(C)
    B, L, k = 5, 77, 31
    y = torch.randn(B, L, C, generator=g).to(torch.bfloat16)
    kept = torch.stack([torch.cat([torch.zeros(1, dtype=torch.long),
                                   torch.sort(torch.randperm(L - 1, generator=g)[:k] + 1).values])
                        for _ in range(B)]).to(torch.int32)
    out = rs.rs_gather_rows(y.to(dev), kept.to(dev), k)
    ref = np.stack([oracle.gather(y[b].float().numpy(), kept[b].numpy()) for b in range(B)])
    assert np.array_equal(out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("L,C,k", [(197, 384, 137), (197, 768, 118), (256, 192, 0), (1, 64, 0),
                                   (50, 2048, 49), (1569, 768, 784)])
def test_select_gather_equals_separate_steps(L, C, k):
    """rs_select_gather (fused for L <= 256) gives the bits of rs_select_topk +
    rs_gather_rows."""
    rs = _rs()
    B = 7
    parts = random_partials(B, L, 4, seed=L + C, ties=(L % 2 == 0)).to(dev)
    g = torch.Generator().manual_seed(k + 1)
    y = torch.randn(B, L, C, generator=g).to(torch.bfloat16).to(dev)
    s1, k1 = rs.rs_select_topk(parts, B, L, k)
    yk1 = rs.rs_gather_rows(y, k1, k)
    s2, k2, yk2 = rs.rs_select_gather(parts, y, k)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2) and torch.equal(k1, k2) and torch.equal(yk1, yk2)


@pytest.mark.parametrize("B,L", [(1, 257), (2, 300), (3, 1098), (16, 1569), (16, 768),
                                 (32, 1569), (5, 4100), (2, 16384), (37, 600)])
@pytest.mark.parametrize("metric,cls", [("l2", True), ("l2", False), ("l1", True),
                                        ("cosine", True), ("cosine", False)])
def test_select_gather_long_sequences(B, L, metric, cls):
    """The fused select+gather on long sequences (radix selection, several CTAs per
    sample when samples are few): the bits of the standalone selection
    (rs_select_topk), the oracle's selection on the same fp32 scores, and the gather
    of the kept rows, on every keep_k edge, with and without ties and a CLS token,
    for each distance."""
    rs = _rs()
    C = 1024 if L <= 1569 else 128
    P = 6 if metric == "cosine" else 8
    nr = L - (1 if cls else 0)
    g = torch.Generator().manual_seed(B * L)
    y = torch.randn(B, L, C, generator=g).to(torch.bfloat16).to(dev)
    for ties in (False, True):
        parts = random_partials(B, L, P, seed=B + L + ties, ties=ties).to(dev)
        for k in sorted({0, 1, nr // 3, nr - 1, nr}):
            s1, k1 = rs.rs_select_topk(parts, B, L, k, distance=metric, cls=cls)
            s2, k2, yk = rs.rs_select_gather(parts, y, k, distance=metric, cls=cls)
            torch.cuda.synchronize()
            assert torch.equal(s1, s2), (B, L, k, "scores")
            assert torch.equal(k1, k2), (B, L, k, "kept_idx")
            s_np = s2.cpu().numpy().astype(np.float64)
            for b in range(B):
                ref = oracle.select_topk(s_np[b], k, cls=cls)
                assert k2[b].cpu().numpy().tolist() == ref.tolist(), (B, L, k, b, "vs oracle")
            ref = torch.stack([y[b][k1[b].long()] for b in range(B)]) if k1.shape[1] else yk
            assert torch.equal(yk, ref), (B, L, k, "y_kept")
    _device_ok()


def _crafted_keys(kind: str, n: int, g: torch.Generator) -> torch.Tensor:
    """fp32 scores shaped to reach each branch of the radix selection."""
    if kind == "all_equal":           # kmin == kmax: no pass at all
        return torch.full((n,), 1.5)
    if kind == "two_values":          # one pass, then bins of hundreds of equal keys
        return torch.where(torch.rand(n, generator=g) < 0.5, torch.tensor(2.0), torch.tensor(3.0))
    if kind == "one_outlier":         # the range is set by one key; the rest tie below it
        v = torch.full((n,), 0.75)
        v[n // 3] = 1e30
        return v
    if kind == "many_binades":        # scores from 2^-60 to 2^60, some exactly zero
        v = torch.pow(2.0, torch.rand(n, generator=g) * 120 - 60)
        v[torch.rand(n, generator=g) < 0.05] = 0.0
        return v
    if kind == "last_bits":           # keys that differ in their last few mantissa bits
        base = torch.tensor(1.0).view(torch.int32).item()
        return (base + torch.randint(0, 100, (n,), generator=g, dtype=torch.int32)).view(torch.float32)
    if kind == "bin_of_32":           # 32 or 33 equal keys straddling the cut, the rest apart
        v = torch.rand(n, generator=g) * 4.0 + 5.0
        v[: n // 2] = torch.rand(n // 2, generator=g) * 0.5 + 0.5
        v[n // 2: n // 2 + 33] = 2.0
        return v
    raise ValueError(kind)


@pytest.mark.parametrize("L", [257, 1569, 4100])
@pytest.mark.parametrize("kind", ["all_equal", "two_values", "one_outlier", "many_binades",
                                  "last_bits", "bin_of_32"])
def test_select_crafted_key_distributions(L, kind):
    """Key sets that drive the radix selection through each of its exits (no pass, the
    full key reached, the final bin of at most 32 keys, bins of exactly 32 and 33): the
    kept lists of the standalone and the fused selection, with and without CLS, at
    every keep_k edge and around the 32-key bin, bit for bit against the oracle on the
    same fp32 scores (L1 with one partial per row, so the score is the partial)."""
    rs = _rs()
    B, C = 3, 128
    g = torch.Generator().manual_seed(L * 7 + len(kind))
    parts = torch.stack([_crafted_keys(kind, L, g) for _ in range(B)]).reshape(B * L, 1)
    pd = parts.to(dev)
    y = torch.randn(B, L, C, generator=g).to(torch.bfloat16).to(dev)
    for cls in (True, False):
        nr = L - (1 if cls else 0)
        half = L // 2 - (1 if cls else 0)
        for k in sorted({0, 1, nr // 3, half - 1, half, half + 31, half + 32, half + 33, nr - 1, nr}):
            if not 0 <= k <= nr:
                continue
            s1, k1 = rs.rs_select_topk(pd, B, L, k, distance="l1", cls=cls)
            s2, k2, yk = rs.rs_select_gather(pd, y, k, distance="l1", cls=cls)
            torch.cuda.synchronize()
            assert torch.equal(s1.cpu().reshape(-1), parts.reshape(-1)), (kind, L, "scores")
            assert torch.equal(k1, k2), (kind, L, k, cls)
            s_np = s1.cpu().numpy().astype(np.float64)
            for b in range(B):
                ref = oracle.select_topk(s_np[b], k, cls=cls)
                assert k1[b].cpu().numpy().tolist() == ref.tolist(), (kind, L, k, cls, b)
            if k2.shape[1]:
                ref_rows = torch.stack([y[b][k2[b].long()] for b in range(B)])
                assert torch.equal(yk, ref_rows), (kind, L, k, cls, "rows")
    _device_ok()


# --------------------------------------------------------------------------- LN stats
@pytest.mark.parametrize("C", [64, 192, 384, 768, 1024, 2048])
def test_ln_stats(C):
    rs = _rs()
    inp = random_block(3, 45, C, 64, seed=C, fg_rows=5)
    x = inp.x.reshape(-1, C)
    st = rs.rs_ln_stats(x.to(dev)).cpu().numpy()
    x64 = parity.f64(x)
    mu = x64.mean(1)
    var = ((x64 - mu[:, None]) ** 2).mean(1)
    assert np.allclose(st[:, 0], mu, rtol=0, atol=1e-5)
    assert np.allclose(st[:, 1], 1 / np.sqrt(var + oracle.EPS), rtol=2e-5, atol=0)


# --------------------------------------------------------------------------- GELU
def test_gelu_apply_error_bound():
    """The epilogue's GELU against the exact z * Phi(z) (fp64 oracle): |error| <= 2e-5 on
    warps whose values all lie in |z| <= 3 (the near-range polynomial, fitted to 1.5e-5:
    the result is stored as bf16, whose half-spacing is >= 9.8e-5 for outputs of
    magnitude >= 0.05) and <= 1.5e-6 on warps holding wider values (the full-range
    one)."""
    rs = _rs()
    g = torch.Generator().manual_seed(2)
    z = torch.cat([torch.linspace(-3, 3, 262144),                 # whole warps in range
                   torch.linspace(-12, 12, 400001),               # mixed warps
                   torch.randn(100000, generator=g) * 0.4,        # hidden-like values
                   torch.tensor([0.0, -0.0, 1e-30, -1e-30, 3.0, -3.0, 5.3, -5.3, 40.0, -40.0])]
                  ).float()
    g = rs.rs_gelu_apply(z.to(dev)).cpu().double().numpy()
    ref = oracle.gelu(z.double().numpy())
    err = np.abs(g - ref)
    assert err.max() <= 2e-5, err.max()
    near = np.arange(z.numel()) < 262144  # the first block: whole warps in |z| <= 3
    assert err[~near][np.abs(z.numpy()[~near]) > 3.2].max() <= 1.5e-6  # full-range warps
    small = np.abs(z.numpy()) < 1e-3
    assert np.all(err[small] <= 2e-5 * np.abs(ref[small]) + 1e-37)


# --------------------------------------------------------------------------- fc1 / fc2
@pytest.mark.parametrize("variant", ["folded", "staged"])
@pytest.mark.parametrize("M,C,H", [(394, 192, 768), (130, 384, 1536), (77, 768, 3072),
                                   (300, 1024, 4096), (1, 64, 64), (129, 128, 192)])
def test_fc1_hidden(M, C, H, variant):
    """a = GELU(LN(x') W1^T + b1) stored as bf16, vs the oracle in fp64: the LN folded
    into the GEMM (default) and the LN staged into the A operand."""
    rs = _rs()
    inp = random_block(1, M, C, H, seed=M + C, fg_rows=M // 4)
    x = inp.x.reshape(M, C)
    w = inp.weights[0]
    fn = rs.rs_ln_fc1_gelu if variant == "folded" else rs.rs_ln_fc1_gelu_staged
    hid = fn(x.to(dev), w.W1.to(dev), w.b1.to(dev), w.gamma.to(dev), w.beta.to(dev))
    w64 = parity.weights64(w)
    ref = oracle.gelu(oracle.fc(oracle.layer_norm(parity.f64(x), w64["gamma"], w64["beta"]),
                                w64["W1"], w64["b1"]))
    parity.check_y(parity.f64(hid), ref, "hidden")
    _device_ok()


def test_fc1_split_steps_equal_combined_step():
    """rs_ln_stats + rs_ln_fold + rs_fc1_gelu_folded launch the same kernels as
    rs_ln_fc1_gelu: identical bits."""
    rs = _rs()
    M, C, H = 333, 384, 1536
    inp = random_block(1, M, C, H, seed=9, fg_rows=30)
    x = inp.x.reshape(M, C).to(dev)
    w = inp.weights[0]
    W1, b1, g, be = (t.to(dev) for t in (w.W1, w.b1, w.gamma, w.beta))
    ref = rs.rs_ln_fc1_gelu(x, W1, b1, g, be)
    stats = rs.rs_ln_stats(x)
    Wg, cg, cc = rs.rs_ln_fold(W1, b1, g, be)
    hid = rs.rs_fc1_gelu_folded(x, stats, Wg, cg, cc)
    torch.cuda.synchronize()
    assert torch.equal(hid, ref)
    # the fold itself: Wg = bf16(W1 * gamma), G = sum_c Wg, cb = W1 beta + b1
    Wg_ref = (w.W1.float() * w.gamma.float()).to(torch.bfloat16)
    assert torch.equal(Wg.cpu(), Wg_ref)
    assert np.allclose(cg.cpu().double().numpy(), Wg_ref.double().sum(1).numpy(), rtol=1e-5, atol=1e-5)
    cb_ref = parity.f64(w.W1) @ parity.f64(w.beta) + parity.f64(w.b1)
    assert np.allclose(cc.cpu().double().numpy(), cb_ref, rtol=1e-4, atol=1e-5)


def test_fc1_large_mean_rows():
    """Rows with a large common offset (mean >> std): the folded LN subtracts
    mean * G after the GEMM, so check it against the oracle on such rows."""
    rs = _rs()
    M, C, H = 256, 768, 1536
    inp = random_block(1, M, C, H, seed=77)
    x = (inp.x.float().reshape(M, C) + torch.linspace(-30, 30, M)[:, None]).to(torch.bfloat16)
    w = inp.weights[0]
    w64 = parity.weights64(w)
    ref = oracle.gelu(oracle.fc(oracle.layer_norm(parity.f64(x), w64["gamma"], w64["beta"]),
                                w64["W1"], w64["b1"]))
    for fn in (rs.rs_ln_fc1_gelu, rs.rs_ln_fc1_gelu_staged):
        hid = fn(x.to(dev), w.W1.to(dev), w.b1.to(dev), w.gamma.to(dev), w.beta.to(dev))
        parity.check_y(parity.f64(hid), ref, fn.__name__)


@pytest.mark.parametrize("M,C,H", [(394, 192, 768), (130, 384, 1536), (77, 768, 3072),
                                   (300, 1024, 4096), (129, 128, 192), (5, 320, 64)])
def test_fc2_residual_shift(M, C, H):
    """y = x' + a W2^T + b2 and the per-row partial sums of (h - x')^2, for a given bf16
    hidden activation a (drawn here; the same a feeds both sides)."""
    rs = _rs()
    inp = random_block(1, M, C, H, seed=M + H, fg_rows=M // 4)
    x = inp.x.reshape(M, C)
    w = inp.weights[0]
    g = torch.Generator().manual_seed(M * 3 + 1)
    a = (torch.randn(M, H, generator=g) * 0.3).to(torch.bfloat16)
    y, parts = rs.rs_fc2_residual_shift(a.to(dev), x.to(dev), w.W2.to(dev), w.b2.to(dev))
    w64 = parity.weights64(w)
    x64 = parity.f64(x)
    h = oracle.fc(parity.f64(a), w64["W2"], w64["b2"])
    parity.check_y(parity.f64(y), h + x64, "y")
    s_ref = oracle.shift_score(h, x64)
    s_gpu = np.sqrt(parts.double().cpu().numpy().sum(1))
    parity.check_scores(s_gpu, s_ref)
    _device_ok()


@pytest.mark.parametrize("M,C,H", [(394, 192, 768), (300, 384, 1536), (130, 384, 1536),
                                   (77, 128, 256), (1, 64, 128), (259, 320, 640), (1000, 256, 512)])
def test_mlp_fused(M, C, H):
    """The fused MLP (fc1, folded LN, GELU, fc2, b2, residual and shift partials with the
    hidden activation kept on chip) vs the oracle in fp64, and vs the two-GEMM path on
    the same LN statistics and folded weights. Widths take both fc2 piece sizes
    (C % 128 == 0 or not) and one to six fc1 k-blocks; M takes ragged last tiles and
    several tiles per CTA."""
    rs = _rs()
    assert rs.rs_mlp_fused_supported(C, H)
    inp = random_block(1, M, C, H, seed=M + 7 * C, fg_rows=M // 4)
    x = inp.x.reshape(M, C)
    w = inp.weights[0]
    xd = x.to(dev)
    W1, b1, W2, b2, g, be = _to_dev(w)
    stats = rs.rs_ln_stats(xd)
    Wg, cg, cc = rs.rs_ln_fold(W1, b1, g, be)
    y, parts = rs.rs_mlp_fused(xd, stats, Wg, cg, cc, W2, b2)
    torch.cuda.synchronize()
    assert parts.shape == (M, rs.RS_FUSED_PARTIALS)
    w64 = parity.weights64(w)
    _, y_ref, s_ref = oracle.sublayer(parity.f64(x), w64["W1"], w64["b1"], w64["W2"],
                                      w64["b2"], w64["gamma"], w64["beta"])
    parity.check_y(parity.f64(y), y_ref, "y (fused)")
    s_gpu = np.sqrt(parts.double().cpu().numpy().sum(1))
    parity.check_scores(s_gpu, s_ref)
    # the two-GEMM path on the same device inputs: the same y and scores up to the
    # fp32 summation order and a bf16 rounding of y
    hid = rs.rs_fc1_gelu_folded(xd, stats, Wg, cg, cc)
    y2, parts2 = rs.rs_fc2_residual_shift(hid, xd, W2, b2)
    torch.cuda.synchronize()
    dy = (y.float() - y2.float()).abs().max().item()
    assert dy <= 2e-2 * max(1.0, y2.float().abs().max().item()), dy
    s2 = np.sqrt(parts2.double().cpu().numpy().sum(1))
    assert np.allclose(s_gpu, s2, rtol=1e-4, atol=1e-6)
    _device_ok()


# --------------------------------------------------------------------------- whole block
def _run_block(x, w, k):
    rs = _rs()
    W = _to_dev(w)
    out = rs.rs_block_forward(x.to(dev), *W, k)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("name", ["tiny_deit_t", "deit_s", "deit_b"])
def test_block_config(name):
    """Full batch on the GPU (the launch bench.py times), every sample checked against
    the oracle: scores, kept_idx (exact where the oracle's k-th and (k+1)-th scores
    are 1e-3 apart, a valid top-k within that band otherwise) and the kept rows of y."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0)
    k = wl.keep_k[0]
    gpu = _run_block(inp.x, inp.weights[0], k)
    ref = parity.oracle_block(inp.x, inp.weights[0], k)
    res = parity.check_block(gpu, ref, k)
    assert res["exact"] + res["band"] == wl.B
    print(name, res)
    _device_ok()


@pytest.mark.parametrize("name", ["umt_b", "umt_l"])
def test_video_config(name):
    """UMT-shaped configs at full batch; 4 sampled clips checked. Each UMT-L stage is
    checked on the oracle's own (bf16-stored) previous-stage output."""
    wl = WORKLOADS[name]
    inp = make_inputs(wl, seed=0)
    samples = [0, 5, 9, wl.B - 1]
    x_gpu = inp.x
    x_ref = inp.x[samples]
    for s in range(wl.stages):
        k = wl.keep_k[s]
        x_in = x_gpu.clone()
        x_in[samples] = x_ref  # checked clips start from the oracle's previous output
        gpu = _run_block(x_in, inp.weights[s], k)
        ref = parity.oracle_block(x_ref, inp.weights[s], k)
        res = parity.check_block(gpu, ref, k, samples)
        print(name, "stage", s, res)
        x_gpu = gpu[0].cpu()
        x_ref = torch.from_numpy(ref[0]).to(torch.bfloat16)
    _device_ok()


# --------------------------------------------------------------------------- edge cases
@pytest.mark.parametrize("B,L,C,H", [(3, 50, 128, 256), (1, 2, 64, 64), (2, 129, 192, 768),
                                     (4, 197, 320, 640), (1, 1, 64, 128)])
def test_block_edges(B, L, C, H):
    """Ragged M (not a multiple of 128), tiny L, odd widths, every keep_k edge."""
    inp = random_block(B, L, C, H, seed=B * L + C, fg_rows=L // 3)
    for k in sorted({0, min(1, L - 1), max(L - 2, 0), L - 1}):
        gpu = _run_block(inp.x, inp.weights[0], k)
        ref = parity.oracle_block(inp.x, inp.weights[0], k)
        parity.check_block(gpu, ref, k)


def test_block_calls_of_changing_shapes():
    """Calls of changing batch and length in a row, on the workspace the previous call
    left, all match the oracle on every sample: 16 long samples (nine select+gather CTAs
    per sample), a short batch, 400 short samples (more select+gather CTAs than fit on
    the GPU at once), and the first shape again."""
    cases = [(16, 300, 128, 256, 200), (3, 41, 128, 256, 20), (400, 9, 64, 128, 5),
             (16, 300, 128, 256, 200)]
    for i, (B, L, C, H, k) in enumerate(cases):
        inp = random_block(B, L, C, H, seed=100 + i, fg_rows=L // 3)
        gpu = _run_block(inp.x, inp.weights[0], k)
        ref = parity.oracle_block(inp.x, inp.weights[0], k)
        parity.check_block(gpu, ref, k)
    _device_ok()


@pytest.mark.parametrize("B,L,C,H", [(2, 65, 2048, 8192), (1, 130, 1024, 16384),
                                     (3, 41, 2048, 2048)])
def test_block_max_widths(B, L, C, H):
    """The widest blocks the library accepts: C = 2048 (the widest LayerNorm row, eight
    16-byte vectors per lane in the gather, CTA-pair GEMMs on both sides) and H = 16384
    (256 k-blocks in fc2), against the oracle on every sample and keep_k edge."""
    inp = random_block(B, L, C, H, seed=B + L + C + H, fg_rows=L // 3)
    for k in (0, L // 2, L - 1):
        gpu = _run_block(inp.x, inp.weights[0], k)
        ref = parity.oracle_block(inp.x, inp.weights[0], k)
        parity.check_block(gpu, ref, k)
    _device_ok()


def test_block_duplicate_rows_tie_rule():
    """Duplicated patch rows give identical scores on both sides; the lower index wins."""
    B, L, C, H = 2, 60, 192, 768
    inp = random_block(B, L, C, H, seed=21, fg_rows=10)
    x = inp.x.clone()
    x[:, 40] = x[:, 7]
    x[:, 41] = x[:, 7]
    x[:, 12] = x[:, 3]
    gpu = _run_block(x, inp.weights[0], 25)
    s = gpu[2].cpu()
    assert torch.equal(s[:, 40], s[:, 7]) and torch.equal(s[:, 41], s[:, 7])
    ref = parity.oracle_block(x, inp.weights[0], 25)
    parity.check_block(gpu, ref, 25)
    for b in range(B):
        kept = gpu[1][b].tolist()
        if 40 in kept:
            assert 7 in kept
        if 41 in kept:
            assert 40 in kept


def test_block_zero_second_layer_closed_form():
    """W2 = 0: h = b2 for every token, so y = x' + b2 (one bf16 rounding) and
    s = ||b2 - x'||; a row equal to b2 scores 0."""
    B, L, C, H = 2, 70, 256, 512
    inp = random_block(B, L, C, H, seed=5)
    w = inp.weights[0]
    w.W2 = torch.zeros_like(w.W2)
    x = inp.x.clone()
    x[1, 9] = w.b2
    gpu = _run_block(x, w, 30)
    y_kept, kept, s = (t.cpu() for t in gpu)
    x64 = parity.f64(x)
    b2 = parity.f64(w.b2)
    s_ref = np.sqrt(((x64 - b2) ** 2).sum(-1))
    assert s[1, 9].item() == 0.0
    assert np.allclose(s.double().numpy(), s_ref, rtol=1e-5, atol=1e-6)
    for b in range(B):
        rows = kept[b].long()
        exp = torch.from_numpy(x64[b][rows.numpy()] + b2).to(torch.bfloat16)
        assert torch.equal(y_kept[b], exp)


def test_block_empty_batch():
    rs = _rs()
    inp = random_block(1, 10, 64, 64, seed=1)
    W = _to_dev(inp.weights[0])
    x = torch.empty(0, 10, 64, dtype=torch.bfloat16, device=dev)
    y_kept, kept, s = rs.rs_block_forward(x, *W, 3)
    assert y_kept.shape == (0, 4, 64)
