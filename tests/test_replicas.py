"""Multi-replica host plumbing with 2 gloo ranks on CPU: per-rank shards, the
max-over-ranks timing and the whole-job throughput (no GPU, no data-path
collective)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from free_vit_token_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import numpy as np

    import oracle
    from workloads import random_block

    w, r, _ = replicas.init("gloo", timeout_s=60)
    assert (w, r) == (world, rank)
    replicas.barrier(w)
    # each replica draws its own shard and computes it with no exchange
    inp = random_block(2, 20, 64, 128, seed=replicas.rank_seed(100, r), fg_rows=3)
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    wt = inp.weights[0]
    _, kept, s, _ = oracle.block_forward(f(inp.x), f(wt.W1), f(wt.b1), f(wt.W2), f(wt.b2),
                                         f(wt.gamma), f(wt.beta), 7)
    elapsed_ms = 10.0 + 5.0 * r  # the slowest rank decides the job time
    mx = replicas.max_over_ranks(elapsed_ms, w)
    thr = replicas.job_throughput(40, 3, mx, w)
    np.save(os.path.join(out_dir, f"r{r}.npy"), np.concatenate([[mx, thr], s.ravel()]))
    replicas.barrier(w)
    replicas.shutdown(w)


def test_two_gloo_replicas(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    import numpy as np

    a = np.load(tmp_path / "r0.npy")
    b = np.load(tmp_path / "r1.npy")
    assert a[0] == b[0] == 15.0                    # max over ranks
    assert a[1] == b[1] == 2 * 40 * 3 / 0.015      # whole-job tokens/s
    assert not np.array_equal(a[2:], b[2:])        # different shards


def test_single_process_defaults():
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_throughput(100, 10, 500.0, 1) == 2000.0
    with pytest.raises(ValueError):
        replicas.job_throughput(1, 1, 0.0, 1)
    assert replicas.rank_seed(7, 3) == 10
