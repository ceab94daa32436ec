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


def _block_args(B, seed):
    wl = WORKLOADS["deit_s"]
    inp = make_inputs(wl, seed=seed, batch=B)
    w = inp.weights[0]
    W = [t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]
    return inp.x.to(dev), W, wl.keep_k[0]


def test_workspace_growth_is_stream_ordered():
    """Growing the workspace does not synchronise the device: the host returns from a
    call that grows it while a long kernel queued on another stream is still running,
    and the grown call's results equal those of a call on an already-grown workspace."""
    rs = _rs()
    x_small, W, k = _block_args(2, seed=5)
    x_big, _, _ = _block_args(64, seed=6)
    s_main, s_other = torch.cuda.Stream(), torch.cuda.Stream()
    rs.rs_release_workspace()
    with torch.cuda.stream(s_main):
        rs.rs_block_forward(x_small, *W, k, stream=s_main)  # a small workspace exists
    torch.cuda.synchronize()
    B, L, C = x_big.shape
    got = (torch.empty(B, k + 1, C, dtype=torch.bfloat16, device=dev),
           torch.empty(B, k + 1, dtype=torch.int32, device=dev),
           torch.empty(B, L, dtype=torch.float32, device=dev))
    torch.cuda.synchronize()
    done = torch.cuda.Event()
    with torch.cuda.stream(s_other):
        torch.cuda._sleep(2_000_000_000)  # about a second of spinning, on its own stream
        done.record(s_other)
    rs.rs_block_forward(x_big, *W, k, *got, stream=s_main)  # grows the workspace
    still_running = not done.query()
    torch.cuda.synchronize()
    assert still_running, "the growing call waited for unrelated work on another stream"
    with torch.cuda.stream(s_main):
        want = rs.rs_block_forward(x_big, *W, k, stream=s_main)  # no growth this time
    torch.cuda.synchronize()
    assert rs.rs_get_last_device_error() == 0
    for a, b in zip(got, want):
        assert torch.equal(a, b)


def test_workspace_cannot_grow_during_capture():
    """A call that would have to grow the workspace while its stream is being captured
    returns RS_ERR_NO_MEM before launching anything; the capture ends cleanly and the
    same call made eagerly afterwards succeeds."""
    rs = _rs()
    x_small, W, k = _block_args(2, seed=7)
    x_big, _, _ = _block_args(32, seed=8)
    s = torch.cuda.Stream()
    rs.rs_release_workspace()
    with torch.cuda.stream(s):
        rs.rs_block_forward(x_small, *W, k, stream=s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    err = None
    with torch.cuda.graph(g, stream=s):
        try:
            rs.rs_block_forward(x_big, *W, k, stream=s)
        except rs.RsError as e:
            err = e
    assert err is not None and err.status == rs.rs.RS_ERR_NO_MEM
    del g
    with torch.cuda.stream(s):
        rs.rs_block_forward(x_big, *W, k, stream=s)
    torch.cuda.synchronize()
    assert rs.rs_get_last_device_error() == 0
