"""Failure detection on the GPU without a fault: a pipeline wait that can never
complete (one k-block load withheld by a test hook) must time out, be reported
as RS_ERR_DEVICE_TIMEOUT through the device flag, and leave the CUDA context
usable. No trap, no hang: every wait in the kernel is time-bounded."""
import pytest
import torch

import oracle
import parity
from workloads import random_block

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,C,H", [(300, 384, 1536),    # single-CTA tiles
                                   (300, 1024, 4096)])  # CTA-pair tiles (K >= 1024)
def test_withheld_load_times_out_and_context_survives(M, C, H):
    import free_vit_token_b200 as rs
    import free_vit_token_b200.rs as rsmod

    dev = torch.device("cuda:0")
    inp = random_block(1, M, C, H, seed=31, fg_rows=20)
    x = inp.x.reshape(M, C).to(dev)
    w = inp.weights[0]
    W1, b1, g, be = (t.to(dev) for t in (w.W1, w.b1, w.gamma, w.beta))
    hid = torch.zeros(M, H, dtype=torch.bfloat16, device=dev)
    assert rs.rs_get_last_device_error() == rsmod.RS_OK
    rs.rs_debug_fc1_skip_load(x, W1, b1, g, be, hid, skip_kblock=2, timeout_us=20000)
    assert rs.rs_get_last_device_error() == rsmod.RS_ERR_DEVICE_TIMEOUT
    assert rs.rs_get_last_device_error() == rsmod.RS_OK  # reading the flag clears it
    # the context still works: the same step without the hook is correct
    out = rs.rs_ln_fc1_gelu(x, W1, b1, g, be)
    torch.cuda.synchronize()
    w64 = parity.weights64(w)
    ref = oracle.gelu(oracle.fc(oracle.layer_norm(parity.f64(x.cpu()), w64["gamma"], w64["beta"]),
                                w64["W1"], w64["b1"]))
    parity.check_y(parity.f64(out), ref, "hidden after timeout")
    assert rs.rs_get_last_device_error() == rsmod.RS_OK


@pytest.mark.parametrize("L,skip", [(300, 2), (64, 0)])
def test_attention_withheld_load_times_out_and_context_survives(L, skip):
    """The attention core's waits are bounded too: one CTA's key tiles withheld from
    block `skip` on, the MMA warp's wait runs out, the flag reads
    RS_ERR_DEVICE_TIMEOUT, and the next ordinary call is correct."""
    import free_vit_token_b200 as rs
    import free_vit_token_b200.rs as rsmod
    from oracle import attn_oracle
    from workloads import random_qkv

    dev = torch.device("cuda:0")
    heads = 2
    qkv = random_qkv(2, L, heads, seed=L).to(dev)
    out = torch.zeros(2, L, 64 * heads, dtype=torch.bfloat16, device=dev)
    assert rs.rs_get_last_device_error() == rsmod.RS_OK
    rs.rs_debug_attn_skip_load(qkv, heads, out, skip_block=skip, timeout_us=20000)
    assert rs.rs_get_last_device_error() == rsmod.RS_ERR_DEVICE_TIMEOUT
    assert rs.rs_get_last_device_error() == rsmod.RS_OK
    got = rs.rs_attn_core(qkv, heads)
    torch.cuda.synchronize()
    q64 = parity.f64(qkv.cpu())
    for b in range(2):
        parity.check_y(parity.f64(got[b].cpu()), attn_oracle.attention_core(q64[b], heads),
                       "attention after timeout")
    assert rs.rs_get_last_device_error() == rsmod.RS_OK


def test_hook_argument_checks():
    import free_vit_token_b200.rs as rsmod

    L = rsmod.lib()
    fake = 0x10000
    assert L.rs_debug_fc1_skip_load(fake, 10, 384, 1536, fake, fake, fake, fake, fake, 6, 1000,
                                    None) == rsmod.RS_ERR_SHAPE
    assert L.rs_debug_fc1_skip_load(fake, 10, 384, 1536, fake, fake, fake, fake, fake, 0, 0,
                                    None) == rsmod.RS_ERR_SHAPE
    assert L.rs_debug_attn_skip_load(fake, 1, 300, 2, fake, 5, 1000, None) == rsmod.RS_ERR_SHAPE
    assert L.rs_debug_attn_skip_load(fake, 1, 300, 2, fake, 0, 0, None) == rsmod.RS_ERR_SHAPE
