"""The native encoder entry point (rs_encoder_forward: attention sublayer, MLP
sublayer, pruning by the MLP's representation shift after chosen layers) against
the fp64 encoder oracle (needs a B200)."""
import pytest
import torch

import parity
from oracle import encoder_oracle
from workloads import draw_attn_weights, random_block

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")


def _rs():
    import free_vit_token_b200 as rs  # deferred: collection must not need a GPU
    return rs


def _layers(depth, C, H, seed):
    out = []
    for l in range(depth):
        a = draw_attn_weights(C, seed=seed + 100 * l)
        m = random_block(1, 2, C, H, seed=seed + 100 * l + 1).weights[0]
        out.append([a.Wqkv, a.bqkv, a.Wo, a.bo, a.gamma, a.beta,
                    m.W1, m.b1, m.W2, m.b2, m.gamma, m.beta])
    return out


def _oracle_layers(layers):
    names = ("Wqkv", "bqkv", "Wo", "bo", "gamma1", "beta1", "W1", "b1", "W2", "b2",
             "gamma2", "beta2")
    return [dict(zip(names, (parity.f64(t) for t in lw))) for lw in layers]


def test_encoder_matches_oracle():
    """Four layers, pruning after layers 1 and 3. With 60 foreground rows (x3) per
    sample the first pruning keeps exactly those (their shift is about three times
    the others'), and the second keeps every remaining patch token, so both sides
    keep the same rows and the outputs compare row by row."""
    rs = _rs()
    B, L, C, H, heads = 2, 197, 128, 512, 2
    inp = random_block(B, L, C, 64, seed=21, fg_rows=60)
    layers = _layers(4, C, H, seed=300)
    keep = [-1, 60, -1, 60]
    got = rs.rs_encoder_forward(inp.x.to(dev), [[t.to(dev) for t in lw] for lw in layers],
                                keep, heads)
    torch.cuda.synchronize()
    assert rs.rs_get_last_device_error() == 0
    ref, kept = encoder_oracle.encoder_forward(parity.f64(inp.x), _oracle_layers(layers), keep,
                                               heads)
    fg = inp.foreground.numpy()
    for b in range(B):
        assert kept[0][b].tolist() == [0] + sorted(int(t) for t in fg[b].nonzero()[0])
    assert got.shape == (B, 61, C)
    parity.check_y(parity.f64(got), ref, "encoder output")


def test_encoder_without_pruning():
    rs = _rs()
    B, L, C, H, heads = 1, 150, 192, 768, 3
    inp = random_block(B, L, C, 64, seed=22)
    layers = _layers(2, C, H, seed=400)
    got = rs.rs_encoder_forward(inp.x.to(dev), [[t.to(dev) for t in lw] for lw in layers],
                                [-1, -1], heads)
    torch.cuda.synchronize()
    ref, _ = encoder_oracle.encoder_forward(parity.f64(inp.x), _oracle_layers(layers), [-1, -1],
                                            heads)
    parity.check_y(parity.f64(got), ref, "encoder output")


def test_encoder_deit_schedule_shapes():
    """The 12-layer DeiT-S schedule (§4.2): 197 tokens -> 158 -> 127 -> 102."""
    rs = _rs()
    B, L, C, H, heads = 4, 197, 384, 1536, 6
    inp = random_block(B, L, C, 64, seed=23, fg_rows=40)
    layers = [[t.to(dev) for t in lw] for lw in _layers(12, C, H, seed=500)]
    keep = encoder_oracle.deit_schedule()
    got = rs.rs_encoder_forward(inp.x.to(dev), layers, keep, heads)
    torch.cuda.synchronize()
    assert got.shape == (B, 102, C)
    assert torch.isfinite(got.float()).all()
    assert rs.rs_get_last_device_error() == 0
