"""Runs the pruned-MLP block on one synthetic workload a few times (for profilers).

    python -m free_vit_token_b200.run_block --workload deit_s --iters 3
    python -m free_vit_token_b200.run_block --workload umt_l --attn --iters 2

Every stage of the workload goes through rs_block_forward on cuda:0; with
--attn, the attention sublayer (rs_attn_sublayer) then runs on the first
stage's pruned output, as the next layer would. The device status flag is
checked at the end.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import free_vit_token_b200 as rs  # noqa: E402
from workloads import WORKLOADS, make_inputs  # noqa: E402


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="deit_s", choices=sorted(WORKLOADS))
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller captures)")
    ap.add_argument("--attn", action="store_true",
                    help="also run the attention sublayer on the pruned tokens")
    a = ap.parse_args()
    wl = WORKLOADS[a.workload]
    inp = make_inputs(wl, seed=0, batch=a.batch)
    dev = torch.device("cuda:0")
    x = inp.x.to(dev)
    W = [[t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)] for w in inp.weights]
    Wa = None
    if a.attn:
        from workloads import draw_attn_weights
        aw = draw_attn_weights(wl.C, seed=1000)
        Wa = [t.to(dev) for t in (aw.Wqkv, aw.bqkv, aw.Wo, aw.bo, aw.gamma, aw.beta)]
    for _ in range(a.iters):
        xs = x
        for s, k in enumerate(wl.keep_k):
            xs = rs.rs_block_forward(xs, *W[s], k)[0]
            if Wa is not None and s == 0:
                rs.rs_attn_sublayer(xs, *Wa, wl.C // 64)
    torch.cuda.synchronize()
    status = rs.rs_get_last_device_error()
    if status != 0:
        print("device error:", rs.status_string(status))
        return 1
    print(f"ok: {a.workload} x{a.iters}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
