"""Pruning on the representation shift through the entire attention block (§3.3
"Operation choice" case (iii)), D(x-hat, x_in) with x-hat = y the block output and
x_in the block input, on the CUDA path against the fp64 oracle (needs a B200)."""
import pytest
import torch

import oracle
import parity
from workloads import draw_attn_weights, random_block

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")


def _rs():
    import free_vit_token_b200 as rs  # deferred: collection must not need a GPU
    return rs


@pytest.mark.parametrize("metric", ["l2", "l1", "cosine"])
@pytest.mark.parametrize("cls", [True, False])
@pytest.mark.parametrize("B,L,C,H", [(2, 197, 192, 768), (2, 150, 384, 1536), (1, 300, 128, 256)])
def test_block_shift(metric, cls, B, L, C, H):
    """Independent x_in and x' (single-CTA and CTA-pair fc2, rank and radix selection),
    every keep_k edge."""
    rs = _rs()
    blk = random_block(B, L, C, H, seed=L + C, fg_rows=L // 4)
    x_in = random_block(B, L, C, 64, seed=L + C + 1, fg_rows=L // 5).x
    w = blk.weights[0]
    W = [t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]
    n = L - (1 if cls else 0)
    for k in sorted({0, 1, n // 2, n}):
        gpu = rs.rs_block_forward_block_shift(x_in.to(dev), blk.x.to(dev), *W, k,
                                              distance=metric, cls=cls)
        torch.cuda.synchronize()
        ref = oracle.block_shift_forward(parity.f64(x_in), parity.f64(blk.x), keep_k=k,
                                         metric=metric, cls=cls, **parity.weights64(w))
        parity.check_block(gpu, ref, k, cls=cls)
    assert rs.rs_get_last_device_error() == 0


def test_block_shift_after_attention():
    """The whole layer: x' = x_in + SA(LN(x_in)) on the GPU, then the MLP block scored on
    D(y, x_in); the oracle takes the same bf16 x' and x_in."""
    rs = _rs()
    B, L, C, H = 2, 197, 384, 1536
    blk = random_block(B, L, C, H, seed=5, fg_rows=40)
    aw = draw_attn_weights(C, seed=6)
    x_in = blk.x.to(dev)
    xp = rs.rs_attn_sublayer(x_in, *[t.to(dev) for t in (aw.Wqkv, aw.bqkv, aw.Wo, aw.bo,
                                                          aw.gamma, aw.beta)], C // 64)
    w = blk.weights[0]
    k = 137
    gpu = rs.rs_block_forward_block_shift(x_in, xp, *[t.to(dev) for t in (w.W1, w.b1, w.W2,
                                                                          w.b2, w.gamma,
                                                                          w.beta)], k)
    torch.cuda.synchronize()
    ref = oracle.block_shift_forward(parity.f64(blk.x), parity.f64(xp.cpu()), keep_k=k,
                                     **parity.weights64(w))
    parity.check_block(gpu, ref, k)
    assert rs.rs_get_last_device_error() == 0
