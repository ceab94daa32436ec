"""B200 (sm_100a) implementation of the pruned-MLP block of Representation Shift.

The compute lives in ``librs.so`` (CUDA kernels behind a C ABI, include/rs.h);
``free_vit_token_b200.rs`` is its ctypes binding.
"""
from .rs import (  # noqa: F401
    DISTANCES,
    RS_DIST_COSINE,
    RS_DIST_L1,
    RS_DIST_L2,
    RS_NO_CLS,
    RsError,
    lib,
    rs_attn_core,
    rs_attn_forward,
    rs_attn_sublayer,
    rs_block_forward,
    rs_block_forward_block_shift,
    rs_encoder_forward,
    rs_fc2_residual_shift,
    rs_debug_attn_skip_load,
    rs_debug_fc1_skip_load,
    rs_fc1_gelu_folded,
    rs_gather_rows,
    rs_gelu_apply,
    rs_get_last_device_error,
    rs_ln_fc1_gelu,
    rs_ln_fold,
    rs_ln_fc1_gelu_noalloc,
    rs_ln_fc1_gelu_staged,
    rs_ln_stats,
    rs_mlp_forward,
    rs_num_partials,
    rs_release_workspace,
    rs_select_gather,
    rs_select_topk,
    rs_workspace_bytes,
    status_string,
)
