"""fp64 CPU oracles (test infrastructure, not the product): the pruned-MLP block
(``rs_oracle``), the attention sublayer (``attn_oracle``) and encoder layers with
pruning between them (``encoder_oracle``).

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.
"""
from .rs_oracle import (  # noqa: F401
    EPS,
    block_forward,
    block_shift_forward,
    fc,
    gather,
    gelu,
    layer_norm,
    mlp,
    select_topk,
    shift_score,
    sublayer,
)
