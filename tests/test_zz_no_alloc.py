"""rs_ln_fc1_gelu_noalloc: the fc1 step for callers that cannot allocate device
memory at call time (e.g. inside CUDA stream capture, or under a framework that
owns all device memory). Its scratch is a static device array inside the
library, so its result must match the allocating rs_ln_fc1_gelu's, call after
call, while the array keeps whatever the previous call left in it.

This file sorts last on purpose so that a run stopping at the first failure has
already run every other test. It also passes when run alone in a fresh process.
"""
import pytest
import torch

import parity
from workloads import random_block

pytestmark = pytest.mark.gpu


def test_noalloc_matches_allocating_entry_point_on_consecutive_calls():
    import free_vit_token_b200 as rs

    dev = torch.device("cuda:0")
    # two calls in a row with different shapes: the second one reuses a scratch
    # array the first one filled (larger M, different C and H)
    for M, C, H, seed in [(1000, 384, 1536, 3), (394, 192, 768, 4), (300, 1024, 4096, 5)]:
        inp = random_block(1, M, C, H, seed=seed, fg_rows=M // 4)
        x = inp.x.reshape(M, C).to(dev)
        w = inp.weights[0]
        W1, b1, g, be = (t.to(dev) for t in (w.W1, w.b1, w.gamma, w.beta))
        out = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
        rs.rs_ln_fc1_gelu_noalloc(x, W1, b1, g, be, out)
        ref = rs.rs_ln_fc1_gelu(x, W1, b1, g, be)
        torch.cuda.synchronize()
        parity.check_y(parity.f64(out), parity.f64(ref), f"noalloc M={M} C={C} H={H}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import free_vit_token_b200.rs as rs

    lib = rs.lib()
    fake = 0x10000  # never dereferenced: the size check returns before any launch
    for M, C, H in [(65537, 64, 64), (128, 2048, 4096)]:
        assert lib.rs_ln_fc1_gelu_noalloc(fake, M, C, H, fake, fake, fake, fake, fake,
                                          None) == rs.RS_ERR_SHAPE
