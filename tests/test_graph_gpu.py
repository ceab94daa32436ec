"""Once the library's buffers have grown to a call's sizes, repeating the call
allocates nothing, so the whole block (and the attention sublayer, and a short
encoder) can be captured in a CUDA graph and replayed with the same results as
eager calls (needs a B200)."""
import pytest
import torch

from workloads import WORKLOADS, draw_attn_weights, make_inputs

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")


def _rs():
    import free_vit_token_b200 as rs  # deferred: collection must not need a GPU
    return rs


def test_block_and_attention_in_a_cuda_graph():
    rs = _rs()
    wl = WORKLOADS["deit_s"]
    inp = make_inputs(wl, seed=3, batch=8)
    w = inp.weights[0]
    W = [t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]
    aw = draw_attn_weights(wl.C, seed=4)
    Wa = [t.to(dev) for t in (aw.Wqkv, aw.bqkv, aw.Wo, aw.bo, aw.gamma, aw.beta)]
    x = inp.x.to(dev)
    k = wl.keep_k[0]
    heads = wl.C // 64
    s = torch.cuda.Stream()
    outs = (torch.empty(8, k + 1, wl.C, dtype=torch.bfloat16, device=dev),
            torch.empty(8, k + 1, dtype=torch.int32, device=dev),
            torch.empty(8, wl.L, dtype=torch.float32, device=dev))
    xo = torch.empty(8, k + 1, wl.C, dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(s):
        # eager: grows the buffers, gives the expected results
        rs.rs_block_forward(x, *W, k, *outs, stream=s)
        rs.rs_attn_sublayer(outs[0], *Wa, heads, out=xo, stream=s)
    torch.cuda.synchronize()
    want = [t.clone() for t in outs] + [xo.clone()]
    for t in list(outs) + [xo]:
        t.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        rs.rs_block_forward(x, *W, k, *outs, stream=s)
        rs.rs_attn_sublayer(outs[0], *Wa, heads, out=xo, stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert rs.rs_get_last_device_error() == 0
    for got, ref in zip(list(outs) + [xo], want):
        assert torch.equal(got, ref)
