"""The synthetic input recipe (CPU only)."""
import torch

from workloads import GRID, WORKLOADS, foreground_layout, make_inputs, random_block


def test_shapes_and_dtypes_tiny():
    w = WORKLOADS["tiny_deit_t"]
    inp = make_inputs(w, seed=0)
    assert inp.x.shape == (2, 197, 192) and inp.x.dtype == torch.bfloat16
    wt = inp.weights[0]
    assert wt.W1.shape == (768, 192) and wt.W2.shape == (192, 768)
    assert wt.b1.shape == (768,) and wt.b2.shape == (192,)
    assert wt.gamma.shape == (192,) and wt.beta.shape == (192,)
    assert inp.foreground.sum(1).tolist() == [40, 40]
    assert not inp.foreground[:, 0].any()


def test_deterministic():
    w = WORKLOADS["tiny_deit_t"]
    a, b = make_inputs(w, seed=0), make_inputs(w, seed=0)
    assert torch.equal(a.x, b.x) and torch.equal(a.weights[0].W1, b.weights[0].W1)
    c = make_inputs(w, seed=1)
    assert not torch.equal(a.x, c.x)


def test_truncation_and_scales():
    inp = random_block(1, 8, 256, 512, seed=3)
    W1 = inp.weights[0].W1.float()
    assert W1.abs().max() <= 0.04 * (1 + 2 ** -8)
    assert 0.015 < W1.std() < 0.02
    g = inp.weights[0].gamma.float()
    assert abs(g.mean() - 1) < 0.02


def test_square_layout():
    g = torch.Generator().manual_seed(5)
    fg = foreground_layout(g, 64, 197, "square")
    for b in range(64):
        idx = torch.nonzero(fg[b]).flatten() - 1
        n = len(idx)
        side = int(round(n ** 0.5))
        assert side * side == n and 6 <= side <= 10
        r, c = idx // GRID, idx % GRID
        assert r.max() - r.min() + 1 == side and c.max() - c.min() + 1 == side


def test_video_square_layout():
    g = torch.Generator().manual_seed(6)
    fg = foreground_layout(g, 4, 1569, "video_square")
    assert not fg[:, 0].any()
    for b in range(4):
        for f in range(8):
            blk = fg[b, 1 + 196 * f: 1 + 196 * (f + 1)].view(GRID, GRID)
            assert blk.sum() == 64
            rows = torch.nonzero(blk.any(1)).flatten()
            cols = torch.nonzero(blk.any(0)).flatten()
            assert len(rows) == 8 and len(cols) == 8
            assert rows.max() - rows.min() == 7


def test_umt_l_stage_weights_differ():
    w = WORKLOADS["umt_l"]
    assert w.stages == 3 and [w.stage_L(s) for s in range(3)] == [1569, 1098, 768]
    inp = make_inputs(w, seed=0, batch=1)
    assert len(inp.weights) == 3
    assert not torch.equal(inp.weights[1].W1, inp.weights[2].W1)
