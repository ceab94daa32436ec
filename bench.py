#!/usr/bin/env python
"""Benchmark of the pruned-MLP block (LN -> fc1 -> GELU -> fc2 + residual +
representation-shift score -> per-sample top-k -> row gather) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl rs|reference]

One step = one pass of the whole path over one batch of the workload (every
stage for the chained UMT-L workload). Prints one JSON line on rank 0.

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events on
the launch stream with an L2 flush before it (outside the events: a 256 MiB
write, then a 256 MiB read of a second buffer so that the write's dirty lines
are written back before the step starts); a barrier and a device synchronise
on both sides of the loop; the max over ranks. Per-kernel durations for the
roofline come from a second event-timed loop over the same kernels, launched
one step-level entry point (one kernel) at a time. `--impl reference` times
the fp64 CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "pruned-MLP-block tokens/sec at 1 B200; % of bf16 tensor peak; select+gather GB/s"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
SG_REPS = 20  # select+gather launches per timing graph


def kernels_per_step(wl) -> int:
    """Kernels rs_block_forward launches per stage: LN prep (statistics + weight
    fold), fc1, fc2 and the fused select+gather (rank select for L <= 256, radix
    select above, both inside the same kernel)."""
    return 4 * wl.stages


# Datasheet figures, reported beside the measured denominators for context only.
DATASHEET_BF16_TF = 2250.0
DATASHEET_HBM_GBS = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ----------------------------------------------------------------------------- ncu traffic
GEMM_SOURCES = ["free_vit_token_b200/csrc/rs_mlp.cu", "free_vit_token_b200/csrc/rs_ptx.cuh",
                "free_vit_token_b200/csrc/rs_gelu.cuh", "free_vit_token_b200/csrc/rs_gelu_poly.h",
                "free_vit_token_b200/csrc/rs_internal.h"]


def gemm_source_hash() -> str:
    """Digest of the GEMM kernels' sources: DRAM traffic measured by ncu is reported
    only while the kernels are the ones that were profiled."""
    import hashlib

    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, stages: int = 1):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from
    profiles/traffic.json, averaged over the workload's stages (one entry per stage,
    as `achieved` averages the stages' launches), or None when an entry is missing
    or was taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    want = gemm_source_hash()
    per_stage = {}
    for e in d.get("entries", []):
        if e.get("kernel") == kernel and e.get("workload") == workload and \
                e.get("source_hash") == want:
            per_stage[int(e.get("stage", 0))] = float(e["dram_bytes_per_launch"])
    if sorted(per_stage) != list(range(stages)):
        return None
    return sum(per_stage.values()) / stages


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.mark_start = None
        self.mark_end = None
        self._lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def _read(self):
        for line in self.proc.stdout:
            self._lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [(t, l) for t, l in self._lines
                if self.mark_start is None or (self.mark_start <= t <= (self.mark_end or 1e30))]
        if not rows:
            rows = self._lines[-5:]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, l in rows:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- dist
from free_vit_token_b200.replicas import (barrier, env_ranks, init as dist_init,  # noqa: E402
                                          job_throughput, max_over_ranks, rank_seed, shutdown)


# ----------------------------------------------------------------------------- oracle leg
_ORACLE_INPUTS = {}


def _oracle_inputs(wl, seed: int):
    """The workload's inputs as the oracle takes them (drawn once per run)."""
    key = (wl.name, seed)
    if key not in _ORACLE_INPUTS:
        inp = make_inputs(wl, seed=seed)
        f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
        weights = [dict(W1=f(w.W1), b1=f(w.b1), W2=f(w.W2), b2=f(w.b2), gamma=f(w.gamma),
                        beta=f(w.beta)) for w in inp.weights]
        _ORACLE_INPUTS[key] = (inp, weights)
    return _ORACLE_INPUTS[key]


def oracle_rate(wl, seed: int, budget_s: float):
    """Oracle tokens/s on a bounded sample of the workload (host cores): whole
    samples (all stages) one at a time, cycling over the batch, until the budget
    is spent (at least one sample)."""
    import oracle
    from threadpoolctl import threadpool_info

    inp, weights = _oracle_inputs(wl, seed)
    t0 = time.time()
    done_tokens, samples = 0, 0
    while samples == 0 or (time.time() - t0) < budget_s:
        b = samples % wl.B
        x = inp.x[b:b + 1].to(torch.float64).numpy()
        for s in range(wl.stages):
            yk, _, _, _ = oracle.block_forward(x, keep_k=wl.keep_k[s], **weights[s])
            done_tokens += x.shape[1]
            x = yk
        samples += 1
    dt = time.time() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return done_tokens / dt, samples, dt, threads


# ----------------------------------------------------------------------------- main
def time_variants(rs, wl, x, W0, out0, dev, stream, reps: int):
    """The first stage's block with the other scores and modes the library offers,
    against the L2 default measured the same way (mean of `reps` back-to-back calls
    between CUDA events, inputs L2-warm): the L1 and cosine distances, no CLS token
    (k + 1 of all L tokens ranked, the same output sizes), the whole-block shift
    D(y, x_in) (x_in: a second [B, L, C] input), and the attention sublayer followed
    by pruning on its own shift."""
    if reps <= 0:
        return None
    from workloads import draw_attn_weights
    k = wl.keep_k[0]
    y_kept, kept, scores = out0
    x_in = torch.flip(x, dims=[1]).contiguous()
    calls = {
        "l2": lambda: rs.rs_block_forward(x, *W0, k, y_kept, kept, scores, stream=stream),
        "l1": lambda: rs.rs_block_forward(x, *W0, k, y_kept, kept, scores, stream=stream,
                                          distance="l1"),
        "cosine": lambda: rs.rs_block_forward(x, *W0, k, y_kept, kept, scores, stream=stream,
                                              distance="cosine"),
        "no_cls": lambda: rs.rs_block_forward(x, *W0, k + 1, y_kept, kept, scores, stream=stream,
                                              cls=False),
        "block_shift": lambda: rs.rs_block_forward_block_shift(x_in, x, *W0, k, y_kept, kept,
                                                               scores, stream=stream),
    }
    if wl.C % 64 == 0:
        aw = draw_attn_weights(wl.C, seed=1001)
        Wa = [t.to(dev) for t in (aw.Wqkv, aw.bqkv, aw.Wo, aw.bo, aw.gamma, aw.beta)]
        calls["attention_shift"] = lambda: rs.rs_attn_forward(x, *Wa, wl.C // 64, k, y_kept,
                                                               kept, scores, stream=stream)
    res = {"reps": reps, "timing": "mean of back-to-back calls between CUDA events, L2-warm"}
    for name, fn in calls.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            fn()
        t1.record(stream)
        torch.cuda.synchronize()
        res[name] = {"ms": t0.elapsed_time(t1) / reps}
    assert rs.rs_get_last_device_error() == 0
    for name in calls:
        res[name]["vs_l2"] = res[name]["ms"] / res["l2"]["ms"]
    return res


def time_attention(rs, wl, x_full, x_kept, peaks, dev, stream, reps: int):
    """The attention sublayer (x + SA(LN(x)), Eq. (5)) that the next layer runs, on
    the stage-0 input (L tokens) and on the pruned block's output (1 + k tokens):
    what the pruning saves downstream. Outside the timed steps; each figure is the
    mean of `reps` back-to-back calls between CUDA events on the launch stream
    (inputs L2-warm), and for the attention core alone its FLOP rate against the
    bf16 peak (4 L^2 C flops per sample: Q K^T and P V)."""
    if reps <= 0 or wl.C % 64:
        return None
    from workloads import draw_attn_weights
    heads = wl.C // 64
    w = draw_attn_weights(wl.C, seed=1000)
    W = [t.to(dev) for t in (w.Wqkv, w.bqkv, w.Wo, w.bo, w.gamma, w.beta)]
    res = {"heads": heads, "head_dim": 64, "reps": reps,
           "timing": "mean of back-to-back calls between CUDA events, inputs L2-warm"}
    for tag, xin in (("full", x_full), ("kept", x_kept)):
        B, L, C = xin.shape
        out = torch.empty_like(xin)
        qkv = torch.randn(B, L, 3 * C, device=dev, dtype=torch.float32).to(torch.bfloat16)
        core_out = torch.empty(B, L, C, dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            rs.rs_attn_sublayer(xin, *W, heads, out=out, stream=stream)
            rs.rs_attn_core(qkv, heads, out=core_out, stream=stream)
        torch.cuda.synchronize()
        t = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        t[0].record(stream)
        for _ in range(reps):
            rs.rs_attn_sublayer(xin, *W, heads, out=out, stream=stream)
        t[1].record(stream)
        t[2].record(stream)
        for _ in range(reps):
            rs.rs_attn_core(qkv, heads, out=core_out, stream=stream)
        t[3].record(stream)
        torch.cuda.synchronize()
        sub_ms = t[0].elapsed_time(t[1]) / reps
        core_ms = t[2].elapsed_time(t[3]) / reps
        core_tf = 4.0 * B * L * L * C / (core_ms / 1e3) / 1e12
        proj_flops = 2.0 * B * L * C * 4 * C
        res[tag] = {"tokens_per_sample": L, "sublayer_ms": sub_ms, "core_ms": core_ms,
                    "core_tflops": core_tf, "core_frac_bf16": core_tf / peaks["bf16"],
                    "sublayer_tflops": (proj_flops + 4.0 * B * L * L * C) / (sub_ms / 1e3) / 1e12}
    assert rs.rs_get_last_device_error() == 0
    res["sublayer_speedup_kept_vs_full"] = res["full"]["sublayer_ms"] / res["kept"]["sublayer_ms"]
    return res


def deit_keep_schedule(L: int, depth: int = 12, layers=(1, 4, 7), ratio: float = 0.2):
    """keep[l]: patch tokens kept after layer l (20% of the patch tokens pruned after
    layers 1, 4 and 7, rounded to the nearest integer), -1 where a layer does not prune."""
    keep = [-1] * depth
    patches = L - 1
    for l in layers:
        patches -= int(math.floor(ratio * patches + 0.5))
        keep[l] = patches
    return keep


def time_encoder_schedule(rs, wl, x, dev, stream, reps: int):
    """A 12-layer encoder of this workload's width (attention sublayer + MLP per layer,
    random ViT-initialised weights) through rs_encoder_forward, with the pruning
    schedule of the DeiT runs and without pruning: images/s of each (mean of `reps`
    calls between CUDA events, after two warm-up calls)."""
    if reps <= 0 or wl.C % 64 or wl.stages != 1 or wl.L != 197:
        return None
    from workloads import draw_attn_weights, draw_weights
    heads = wl.C // 64
    layers = []
    for l in range(12):
        a = draw_attn_weights(wl.C, seed=2000 + l)
        m = draw_weights(torch.Generator().manual_seed(3000 + l), wl.C, wl.H)
        layers.append([t.to(dev) for t in (a.Wqkv, a.bqkv, a.Wo, a.bo, a.gamma, a.beta,
                                           m.W1, m.b1, m.W2, m.b2, m.gamma, m.beta)])
    res = {"depth": 12, "heads": heads, "batch": wl.B, "reps": reps,
           "timing": "mean of back-to-back calls between CUDA events"}
    for tag, keep in (("pruned", deit_keep_schedule(wl.L)), ("unpruned", [-1] * 12)):
        for _ in range(2):
            out = rs.rs_encoder_forward(x, layers, keep, heads, stream=stream)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(reps):
            rs.rs_encoder_forward(x, layers, keep, heads, out=out, stream=stream)
        t1.record(stream)
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / reps
        res[tag] = {"keep": keep, "ms": ms, "images_per_s": wl.B / (ms / 1e3),
                    "tokens_out": int(out.shape[1])}
    assert rs.rs_get_last_device_error() == 0
    res["speedup_pruned_vs_unpruned"] = res["unpruned"]["ms"] / res["pruned"]["ms"]
    return res


class Block:
    """One workload's device inputs and outputs for rs_block_forward (every stage)."""

    def __init__(self, rs, wl, seed: int, dev, stream):
        self.rs, self.wl, self.dev, self.stream = rs, wl, dev, stream
        self.inp = make_inputs(wl, seed=seed)
        self.x = self.inp.x.to(dev)
        self.W = [[t.to(dev) for t in (w.W1, w.b1, w.W2, w.b2, w.gamma, w.beta)]
                  for w in self.inp.weights]
        self.outs = [(torch.empty(wl.B, k + 1, wl.C, dtype=torch.bfloat16, device=dev),
                      torch.empty(wl.B, k + 1, dtype=torch.int32, device=dev),
                      torch.empty(wl.B, wl.stage_L(s), dtype=torch.float32, device=dev))
                     for s, k in enumerate(wl.keep_k)]

    def step(self, x0=None, last=None):
        """One pass of the block (every stage); `last` replaces the last stage's outputs."""
        wl = self.wl
        xs = self.x if x0 is None else x0
        for s, k in enumerate(wl.keep_k):
            o = last if (last is not None and s == wl.stages - 1) else self.outs[s]
            self.rs.rs_block_forward(xs, *self.W[s], k, *o, stream=self.stream)
            xs = o[0]


def time_steps(blk, steps: int, warmup: int, l2_flush, world: int, clocks=None):
    """W warm-up steps, then `steps` steps each between CUDA events with an L2 flush
    before it (outside the events); barrier + synchronise around the loop; the max
    over ranks of the summed step times (ms)."""
    for _ in range(warmup):
        l2_flush()
        blk.step()
    torch.cuda.synchronize()
    st = blk.rs.rs_get_last_device_error()
    assert st == 0, blk.rs.status_string(st)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.mark_start = time.time()
    for i in range(steps):
        l2_flush()
        ev[i][0].record(blk.stream)
        blk.step()
        ev[i][1].record(blk.stream)
    torch.cuda.synchronize()
    barrier(world)
    if clocks is not None:
        clocks.mark_end = time.time()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world, blk.dev)
    st = blk.rs.rs_get_last_device_error()
    assert st == 0, blk.rs.status_string(st)
    return total_ms


KERNELS = ("stats", "fold", "fc1", "fc2", "select_gather")


def kernel_breakdown(blk, nrep: int, l2_flush):
    """Each kernel of the block launched through its own step-level entry point between
    CUDA events on the launch stream, after an L2 flush per chain: mean ms per launch,
    per stage. Returns (per_stage {s: {kernel: ms}}, scratch buffers holding the last
    stage-by-stage y and partials as fc2 left them)."""
    rs, wl, dev, stream = blk.rs, blk.wl, blk.dev, blk.stream
    M0 = wl.tokens(0)
    np_ = rs.rs_num_partials(wl.C)
    buf = dict(stats=torch.empty(M0, 2, dtype=torch.float32, device=dev),
               Wg=torch.empty(wl.H, wl.C, dtype=torch.bfloat16, device=dev),
               colG=torch.empty(wl.H, dtype=torch.float32, device=dev),
               colC=torch.empty(wl.H, dtype=torch.float32, device=dev),
               hid=torch.empty(M0 * wl.H, dtype=torch.bfloat16, device=dev),
               y=[torch.empty(wl.tokens(s) * wl.C, dtype=torch.bfloat16, device=dev)
                  for s in range(wl.stages)],
               parts=[torch.empty(wl.tokens(s) * np_, dtype=torch.float32, device=dev)
                      for s in range(wl.stages)])
    recs = []
    for _ in range(nrep):
        l2_flush()
        xs = blk.x
        for s, k in enumerate(wl.keep_k):
            L_s = wl.stage_L(s)
            M = wl.B * L_s
            e = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
            x2 = xs.reshape(M, wl.C)
            st2 = buf["stats"][:M]
            h2 = buf["hid"][: M * wl.H].view(M, wl.H)
            y2 = buf["y"][s].view(M, wl.C)
            p2 = buf["parts"][s].view(M, np_)
            W = blk.W[s]
            o = blk.outs[s]
            e[0].record(stream)
            rs.rs_ln_stats(x2, stats=st2, stream=stream)
            e[1].record(stream)
            rs.rs_ln_fold(W[0], W[1], W[4], W[5], buf["Wg"], buf["colG"], buf["colC"],
                          stream=stream)
            e[2].record(stream)
            rs.rs_fc1_gelu_folded(x2, st2, buf["Wg"], buf["colG"], buf["colC"], hidden=h2,
                                  stream=stream)
            e[3].record(stream)
            rs.rs_fc2_residual_shift(h2, x2, W[2], W[3], y=y2, partials=p2, stream=stream)
            e[4].record(stream)
            rs.rs_select_gather(p2, y2.view(wl.B, L_s, wl.C), k, scores=o[2], kept_idx=o[1],
                                y_kept=o[0], stream=stream)
            e[5].record(stream)
            recs.append((s, e))
            xs = o[0]
    torch.cuda.synchronize()
    per_stage = {}
    for s, e in recs:
        d = per_stage.setdefault(s, {n: [] for n in KERNELS})
        for j, n in enumerate(KERNELS):
            d[n].append(e[j].elapsed_time(e[j + 1]))
    return {s: {n: statistics.mean(v) for n, v in d.items()} for s, d in per_stage.items()}, buf


def select_gather_times(blk, buf, flush_w, flush_r):
    """Device time of one select+gather launch per stage, summed over stages (ms):
    (L2-hot: SG_REPS launches captured in a CUDA graph and replayed, on the partials
    and y fc2 just wrote; after an L2 flush: graph [flush, select+gather] minus graph
    [flush], median of 7)."""
    rs, wl, dev, stream = blk.rs, blk.wl, blk.dev, blk.stream
    np_ = rs.rs_num_partials(wl.C)
    hot, cold = 0.0, 0.0
    per_stage = []  # (hot ms, flushed ms) of each stage's launch
    cap_stream = torch.cuda.Stream(dev)
    for s, k in enumerate(wl.keep_k):
        L_s = wl.stage_L(s)
        M = wl.B * L_s
        y2 = buf["y"][s].view(wl.B, L_s, wl.C)
        p2 = buf["parts"][s].view(M, np_)
        o = blk.outs[s]

        def sg(st):
            rs.rs_select_gather(p2, y2, k, scores=o[2], kept_idx=o[1], y_kept=o[0], stream=st)

        cap_stream.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            for _ in range(SG_REPS):
                sg(cap_stream)
        g.replay()  # replays run on the current stream (`stream`)
        torch.cuda.synchronize()
        reps = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            reps.append(a.elapsed_time(b) / SG_REPS)
        hot_s = statistics.median(reps)
        hot += hot_s
        del g
        gf, gfs = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf, stream=cap_stream):
            flush_w.zero_()
            flush_r.sum()
        with torch.cuda.graph(gfs, stream=cap_stream):
            flush_w.zero_()
            flush_r.sum()
            sg(cap_stream)
        diffs = []
        for _ in range(7):
            tt = []
            for g_ in (gf, gfs):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g_.replay()
                b.record(stream)
                torch.cuda.synchronize()
                tt.append(a.elapsed_time(b))
            diffs.append(tt[1] - tt[0])
        cold_s = max(statistics.median(diffs), 1e-6)
        cold += cold_s
        per_stage.append((hot_s, cold_s))
        del gf, gfs
    st = rs.rs_get_last_device_error()
    assert st == 0, rs.status_string(st)
    return hot, cold, per_stage


def select_gather_stage_bytes(rs, wl, s: int) -> int:
    """Algorithmic bytes of one stage's select+gather: the partials and the scores once,
    kept_idx written, the kept rows read and written."""
    np_ = rs.rs_num_partials(wl.C)
    M, k = wl.tokens(s), wl.keep_k[s]
    return (M * np_ * 4 + M * 4 + wl.B * (k + 1) * 4      # select: partials in, scores + idx out
            + wl.B * (k + 1) * (4 + 2 * wl.C * 2))        # gather: idx in, rows in + out


def select_gather_bytes(rs, wl) -> int:
    """Algorithmic bytes of select+gather over every stage."""
    return sum(select_gather_stage_bytes(rs, wl, s) for s in range(len(wl.keep_k)))


def measure_block(blk, steps: int, warmup: int, l2_flush, flush_w, flush_r, world: int, peaks,
                  clocks=None):
    """The block's timed steps, its kernel breakdown, the GEMM roofline and the
    select+gather bandwidth for one workload."""
    rs, wl = blk.rs, blk.wl
    tokens_per_step = sum(wl.tokens(s) for s in range(wl.stages))
    total_ms = time_steps(blk, steps, warmup, l2_flush, world, clocks)
    ms_per_step = total_ms / steps
    per_stage, buf = kernel_breakdown(blk, max(10, min(steps, 200)), l2_flush)
    kernel_ms = {n: sum(per_stage[s][n] for s in per_stage) for n in KERNELS}
    gemm_flops = sum(2.0 * wl.tokens(s) * wl.C * wl.H for s in range(wl.stages))
    fc = {}
    for n in ("fc1", "fc2"):
        tf = gemm_flops / (kernel_ms[n] / 1e3) / 1e12
        fc[n] = {"ms": kernel_ms[n], "tflops": tf, "frac": tf / peaks["bf16"],
                 "traffic": ncu_traffic(n, wl.name, wl.stages)}
    dominant = max(("fc1", "fc2"), key=lambda n: kernel_ms[n])
    hot, cold, sg_stages = select_gather_times(blk, buf, flush_w, flush_r)
    sg_bytes = select_gather_bytes(rs, wl)
    block_flops = 2.0 * gemm_flops
    block_tf = block_flops / (ms_per_step / 1e3) / 1e12
    gbs = lambda ms: sg_bytes / (ms / 1e3) / 1e9  # noqa: E731
    return {
        "total_ms": total_ms, "ms_per_step": ms_per_step,
        "tokens_per_step": tokens_per_step, "dominant": dominant, "fc": fc,
        "kernel_ms": kernel_ms,
        "kernel_ms_per_stage": {str(s): per_stage[s] for s in per_stage} if wl.stages > 1
        else None,
        "block_tflops": block_tf, "block_frac_of_bf16_peak": block_tf / peaks["bf16"],
        "block_frac_other_peaks": {"bf16_sustained": block_tf / peaks["bf16_sustained"],
                                   "bf16_datasheet_2250": block_tf / DATASHEET_BF16_TF},
        "select_gather": {
            "GBps": gbs(cold), "frac_hbm": gbs(cold) / peaks["hbm"], "bytes": sg_bytes,
            "ms": cold, "frac_of_8TBps": gbs(cold) / DATASHEET_HBM_GBS,
            "timing": "device time per launch right after a 256 MiB L2 flush: graph [flush, "
                      "select+gather] minus graph [flush], median of 7, summed over stages",
            "ms_single_launch_events": kernel_ms["select_gather"],
            "l2_hot": {"ms": hot, "GBps": gbs(hot), "frac_hbm": gbs(hot) / peaks["hbm"],
                       "timing": f"device time per launch, {SG_REPS} launches replayed from a "
                                 "CUDA graph, inputs as fc2 left them (L2-resident)"},
            "per_stage": [
                {"stage": i, "bytes": select_gather_stage_bytes(rs, wl, i),
                 "ms": c, "frac_hbm": select_gather_stage_bytes(rs, wl, i) / (c / 1e3) / 1e9
                 / peaks["hbm"],
                 "l2_hot_ms": h, "l2_hot_frac_hbm": select_gather_stage_bytes(rs, wl, i)
                 / (h / 1e3) / 1e9 / peaks["hbm"]}
                for i, (h, c) in enumerate(sg_stages)] if wl.stages > 1 else None},
    }


def time_e2e(blk, steps: int, l2_flush, world: int):
    """End to end through the public call with host buffers: every step copies its input
    x' from pinned host memory and its outputs (y_kept, kept_idx, scores) back to pinned
    host memory. Steps are pipelined as a serving loop would run them: the H2D copy of
    step i+1 and the D2H copy of step i-1 run on their own streams while step i computes
    (two device buffers for the input and for the outputs). Returns (ms per step, H2D
    bytes, D2H bytes)."""
    dev, stream = blk.dev, blk.stream
    x_h = blk.inp.x.pin_memory()
    h2d = x_h.numel() * x_h.element_size()
    outs_h = tuple(torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in blk.outs[-1])
    d2h = sum(o.numel() * o.element_size() for o in outs_h)
    x_d = [torch.empty_like(blk.x) for _ in range(2)]
    outs_d = [tuple(torch.empty_like(o) for o in blk.outs[-1]) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, comp_done, d2h_done = [], [], []
    barrier(world)
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    s_h2d.wait_stream(stream)
    s_d2h.wait_stream(stream)
    for i in range(steps):
        j = i & 1
        if i >= 2:
            s_h2d.wait_event(comp_done[i - 2])  # step i-2 has read x_d[j]
        with torch.cuda.stream(s_h2d):
            x_d[j].copy_(x_h, non_blocking=True)
        h2d_done.append(ev())
        h2d_done[-1].record(s_h2d)
        stream.wait_event(h2d_done[i])
        if i >= 2:
            stream.wait_event(d2h_done[i - 2])  # outs_d[j] has reached the host
        l2_flush()
        blk.step(x_d[j], last=outs_d[j])
        comp_done.append(ev())
        comp_done[-1].record(stream)
        s_d2h.wait_event(comp_done[i])
        with torch.cuda.stream(s_d2h):
            for oh, od in zip(outs_h, outs_d[j]):
                oh.copy_(od, non_blocking=True)
        d2h_done.append(ev())
        d2h_done[-1].record(s_d2h)
    stream.wait_event(d2h_done[-1])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(t_start.elapsed_time(t_end), world, dev) / steps, h2d, d2h


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="umt_l", choices=sorted(WORKLOADS))
    ap.add_argument("--also", default="deit_b",
                    help="second workload measured in the same run and reported under its "
                         "own key ('' or 'none': skip)")
    ap.add_argument("--impl", default="rs", choices=["rs", "reference"])
    ap.add_argument("--variant-reps", type=int, default=20,
                    help="calls per score-variant timing (0: skip that measurement)")
    ap.add_argument("--encoder-reps", type=int, default=5,
                    help="calls per 12-layer encoder timing (0: skip that measurement)")
    ap.add_argument("--attn-reps", type=int, default=20,
                    help="calls per attention-sublayer timing (0: skip that measurement)")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work for the cpu_baseline leg (0 = skip)")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    also = None if args.also in ("", "none", args.workload) else WORKLOADS[args.also]
    # the reference arm runs on rank 0 alone and joins no process group
    world, rank, local = dist_init("nccl") if args.impl == "rs" else env_ranks()
    tokens_per_step = sum(wl.tokens(s) for s in range(wl.stages))
    config = {"workload": wl.name, "B": wl.B, "L": wl.L, "C": wl.C, "H": wl.H,
              "keep_k": list(wl.keep_k), "stages": wl.stages,
              "tokens_per_step": tokens_per_step, "parallelism": f"replicas{world}",
              "l2": "flushed before every timed step: 256 MiB write + 256 MiB read"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        # per-step sample sized so that the whole run stays near 2.5 minutes of CPU work
        budget = max(0.2, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
        for _ in range(args.warmup):
            oracle_rate(wl, 0, budget / 4)
        rates = []
        info = None
        for _ in range(args.steps):
            r, n, dt, thr = oracle_rate(wl, 0, budget)
            rates.append(r)
            info = (n, dt, thr)
        v = float(np.mean(rates))
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1000.0 * tokens_per_step / v, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": config,
                "cpu_baseline": {"value": v, "unit": UNIT, "cores": info[2], "kind": "oracle",
                                 "sample": f"{info[0]} samples per step (~{info[1]:.1f} s), "
                                           f"workload {wl.name}"},
                "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import free_vit_token_b200 as rs

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    blk = Block(rs, wl, rank_seed(0, rank), dev, stream)
    flush_w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def l2_flush():
        flush_w.zero_()
        flush_r.sum()

    clocks = ClockSampler(local)
    clocks.start()
    m = measure_block(blk, args.steps, args.warmup, l2_flush, flush_w, flush_r, world, peaks,
                      clocks)
    ms_per_step = m["ms_per_step"]
    value = job_throughput(tokens_per_step, args.steps, m["total_ms"], world)
    n_e2e = max(5, min(args.steps, 100))
    e2e_ms, h2d, d2h = time_e2e(blk, n_e2e, l2_flush, world)
    e2e_value = job_throughput(tokens_per_step, 1, e2e_ms, world)
    clocks.stop()

    second = None
    if also is not None:
        b2 = Block(rs, also, rank_seed(0, rank), dev, stream)
        steps2 = max(5, min(args.steps, 50))
        m2 = measure_block(b2, steps2, max(3, min(args.warmup, 10)), l2_flush, flush_w, flush_r,
                           world, peaks)
        second = {"workload": also.name, "B": also.B, "L": also.L, "C": also.C, "H": also.H,
                  "keep_k": list(also.keep_k), "steps": steps2,
                  "tokens_per_s": job_throughput(m2["tokens_per_step"], steps2, m2["total_ms"],
                                                 world),
                  "images_per_s": world * also.B / (m2["ms_per_step"] / 1e3),
                  **{k: v for k, v in m2.items() if k not in ("total_ms", "dominant")}}
        sched = time_encoder_schedule(rs, also, b2.x, dev, stream, args.encoder_reps)
        if sched is not None:
            second["encoder_schedule"] = sched
        del b2

    variants = time_variants(rs, wl, blk.x, blk.W[0], blk.outs[0], dev, stream, args.variant_reps)
    attn = time_attention(rs, wl, blk.x, blk.outs[0][0], peaks, dev, stream, args.attn_reps)
    sched = time_encoder_schedule(rs, wl, blk.x, dev, stream, args.encoder_reps)

    cpu = None
    if rank == 0 and args.cpu_budget > 0:
        r, n, dt, thr = oracle_rate(wl, 0, args.cpu_budget)
        cpu = {"value": r, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": f"{n} samples of {wl.name} (all stages, one sample at a time) in "
                         f"{dt:.1f} s on the host, fp64 numpy/BLAS"}

    dom = m["dominant"]
    fcd = m["fc"][dom]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config,
        "roofline": {"bound": "tensor", "kernel": f"{dom} (tcgen05 GEMM)",
                     "achieved": fcd["tflops"], "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": fcd["frac"], "traffic": fcd["traffic"],
                     "peak_source": f"{peaks['source']} bf16 burst",
                     "kernel_ms": fcd["ms"],
                     "per_launch": "flops and time summed over the workload's stages; "
                                   "traffic averaged over the stages' launches"},
        "gemm_roofline": m["fc"],
        "block_tflops": m["block_tflops"],
        "block_frac_of_bf16_peak": m["block_frac_of_bf16_peak"],
        "block_frac_other_peaks": m["block_frac_other_peaks"],
        "kernel_ms": m["kernel_ms"],
        "kernel_ms_per_stage": m["kernel_ms_per_stage"],
        "select_gather": m["select_gather"],
        "images_per_s": world * wl.B / (ms_per_step / 1e3),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipelining": "H2D of step i+1 and D2H of step i-1 overlap step i (own streams)"},
        "also": second,
        "score_variants": variants,
        "attention_next_layer": attn,
        "encoder_schedule": sched,
        "gpu_launches": kernels_per_step(wl) * args.steps,
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    rs.rs_release_workspace()
    shutdown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
