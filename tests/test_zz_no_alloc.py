"""rs_ln_fc1_gelu_noalloc: the fc1 step for callers that cannot allocate device
memory when they call -- a framework that owns all device memory through its own
pool and forbids other allocations, or latency-bound code that cannot afford a
cudaMalloc/cudaFree, which may synchronise the whole device. Its scratch is a
static device array inside the library that every call shares and that keeps
whatever the previous call left in it.

Checked through the C ABI, call after call with different shapes: against the
fp64 oracle under the parity rule; bit for bit against the allocating
rs_ln_fc1_gelu where both run the same single-CTA kernel (C < 1024; at C = 1024
the allocating path uses CTA pairs, so there the rule is the parity tolerance);
at the exact scratch limits; with the status slot clear afterwards.

This file sorts last on purpose so that a run stopping at the first failure has
already run every other test. It also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from workloads import random_block

pytestmark = pytest.mark.gpu

dev = torch.device("cuda:0")


def _oracle_hidden(x, w, rows=None):
    w64 = parity.weights64(w)
    x64 = parity.f64(x if rows is None else x[rows])
    return oracle.gelu(oracle.fc(oracle.layer_norm(x64, w64["gamma"], w64["beta"]),
                                 w64["W1"], w64["b1"]))


def _run_both(M, C, H, seed):
    import free_vit_token_b200 as rs

    inp = random_block(1, M, C, H, seed=seed, fg_rows=M // 4)
    x = inp.x.reshape(M, C)
    w = inp.weights[0]
    xd = x.to(dev)
    W1, b1, g, be = (t.to(dev) for t in (w.W1, w.b1, w.gamma, w.beta))
    out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    rs.rs_ln_fc1_gelu_noalloc(xd, W1, b1, g, be, out)
    ref = rs.rs_ln_fc1_gelu(xd, W1, b1, g, be)
    torch.cuda.synchronize()
    return x, w, out.cpu(), ref.cpu()


def test_noalloc_matches_oracle_and_allocating_path_on_consecutive_calls():
    import free_vit_token_b200 as rs

    # consecutive calls with different shapes: each call reuses a scratch array the
    # previous one filled (larger M, different C and H)
    for M, C, H, seed in [(1000, 384, 1536, 3), (394, 192, 768, 4), (300, 1024, 4096, 5),
                          (77, 768, 3072, 6)]:
        x, w, out, ref = _run_both(M, C, H, seed)
        what = f"noalloc M={M} C={C} H={H}"
        parity.check_y(parity.f64(out), _oracle_hidden(x, w), what + " vs oracle")
        if C < 1024:
            assert torch.equal(out, ref), what + ": bits differ from rs_ln_fc1_gelu"
        else:
            parity.check_y(parity.f64(out), parity.f64(ref), what + " vs rs_ln_fc1_gelu")
    assert rs.rs_get_last_device_error() == 0


@pytest.mark.parametrize("M,C,H", [(65536, 256, 1024), (128, 1024, 4096)])
def test_noalloc_at_its_limits(M, C, H):
    """Exactly at the scratch limits (M = 65536 rows; H * C = 4194304 folded weights),
    where a wrong offset inside the array would overwrite another region."""
    import free_vit_token_b200 as rs

    x, w, out, ref = _run_both(M, C, H, seed=M + C)
    rows = np.random.default_rng(0).choice(M, 256, replace=False) if M > 4096 else None
    got = parity.f64(out if rows is None else out[rows])
    parity.check_y(got, _oracle_hidden(x, w, rows), f"noalloc M={M} C={C} H={H}")
    if C < 1024:
        assert torch.equal(out, ref)
    else:
        parity.check_y(parity.f64(out), parity.f64(ref), "vs rs_ln_fc1_gelu")
    assert rs.rs_get_last_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import free_vit_token_b200.rs as rs

    lib = rs.lib()
    fake = 0x10000  # never dereferenced: the size check returns before any launch
    for M, C, H in [(65537, 64, 64), (128, 2048, 4096), (64, 1024, 4160)]:
        assert lib.rs_ln_fc1_gelu_noalloc(fake, M, C, H, fake, fake, fake, fake, fake,
                                          None) == rs.RS_ERR_SHAPE
