"""fp64 CPU oracle for the pruned-MLP block (test infrastructure, not the product).

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.
"""
from .rs_oracle import (  # noqa: F401
    EPS,
    block_forward,
    block_shift_forward,
    fc,
    finalize_scores_f32,
    gather,
    gelu,
    layer_norm,
    mlp,
    select_topk,
    shift_score,
    sublayer,
)
