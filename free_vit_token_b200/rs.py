"""ctypes binding of librs.so (see include/rs.h): argument marshalling only.

Every function here forwards torch tensors' device pointers and sizes to the C
entry point of the same name and raises ``RsError`` on a non-zero status. All
arithmetic runs in the library's CUDA kernels; there is no other code path, and
a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librs.so")

RS_OK = 0
RS_ERR_NULL = 1
RS_ERR_SHAPE = 2
RS_ERR_KEEP_K = 3
RS_ERR_ALIGN = 4
RS_ERR_CUDA = 5
RS_ERR_DEVICE_TIMEOUT = 6
RS_ERR_NO_MEM = 7

_vp, _i, _fp, _ip = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
SIGNATURES = {
    "rs_block_forward": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _ip,
                              _fp, _vp]),
    "rs_ln_stats": (_i, [_vp, _i, _i, _fp, _vp]),
    "rs_ln_fc1_gelu": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rs_ln_fc1_gelu_staged": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rs_gelu_apply": (_i, [_fp, _fp, _i, _vp]),
    "rs_debug_fc1_skip_load": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _vp]),
    "rs_ln_fold": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp, _fp, _fp, _vp]),
    "rs_fc1_gelu_folded": (_i, [_vp, _fp, _vp, _fp, _fp, _i, _i, _i, _vp, _vp]),
    "rs_ln_fc1_gelu_noalloc": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rs_fc2_residual_shift": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _fp, _vp]),
    "rs_fc2_residual_shift_ex": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _i, _vp, _fp, _vp]),
    "rs_num_partials_ex": (_i, [_i, _i]),
    "rs_block_forward_ex": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i,
                                 _vp, _ip, _fp, _vp]),
    "rs_select_topk_ex": (_i, [_fp, _i, _i, _i, _i, _i, _i, _fp, _ip, _vp]),
    "rs_select_gather_ex": (_i, [_fp, _i, _vp, _i, _i, _i, _i, _i, _i, _fp, _ip, _vp, _vp]),
    "rs_num_partials": (_i, [_i]),
    "rs_select_topk": (_i, [_fp, _i, _i, _i, _i, _fp, _ip, _vp]),
    "rs_gather_rows": (_i, [_vp, _i, _i, _i, _ip, _i, _vp, _vp]),
    "rs_select_gather": (_i, [_fp, _i, _vp, _i, _i, _i, _i, _fp, _ip, _vp, _vp]),
    "rs_block_forward_block_shift_ex": (_i, [_vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp,
                                             _vp, _i, _i, _i, _vp, _ip, _fp, _vp]),
    "rs_mlp_forward": (_i, [_vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rs_attn_core": (_i, [_vp, _i, _i, _i, _vp, _vp]),
    "rs_debug_attn_skip_load": (_i, [_vp, _i, _i, _i, _vp, _i, _i, _vp]),
    "rs_encoder_forward": (_i, [_vp, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp),
                                ctypes.POINTER(_i), _vp, _vp]),
    "rs_attn_sublayer": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rs_attn_forward_ex": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i,
                                _vp, _ip, _fp, _vp]),
    "rs_mlp_fused_supported": (_i, [_i, _i]),
    "rs_mlp_fused": (_i, [_vp, _fp, _vp, _fp, _fp, _i, _i, _i, _vp, _vp, _vp, _fp, _vp]),
    "rs_status_string": (ctypes.c_char_p, [_i]),
    "rs_get_last_device_error": (_i, [_vp]),
    "rs_release_workspace": (None, []),
    "rs_workspace_bytes": (ctypes.c_uint64, [_i, _i, _i, _i]),
}

_lib = None


class RsError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded librs.so. Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m free_vit_token_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().rs_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != RS_OK:
        raise RsError(status, where)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr() or None


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream or None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream or None
    return int(stream) or None


RS_DIST_L2, RS_DIST_L1, RS_DIST_COSINE = 0, 1, 2
RS_NO_CLS = 1
DISTANCES = {"l2": RS_DIST_L2, "l1": RS_DIST_L1, "cosine": RS_DIST_COSINE}


def _dist(distance) -> int:
    return DISTANCES[distance] if isinstance(distance, str) else int(distance)


def rs_block_forward(x: torch.Tensor, W1, b1, W2, b2, gamma, beta, keep_k: int,
                     y_kept: Optional[torch.Tensor] = None, kept_idx: Optional[torch.Tensor] = None,
                     scores: Optional[torch.Tensor] = None, stream=None, distance="l2",
                     cls: bool = True) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """x [B, L, C] bf16 -> (y_kept [B, n, C] bf16, kept_idx [B, n] int32, scores [B, L] fp32)
    with n = 1 + k (CLS first) or k (cls=False: all L tokens ranked). `distance`: "l2",
    "l1" or "cosine" (or an RS_DIST_* value)."""
    B, L, C = x.shape
    H = W1.shape[0]
    dev = x.device
    n = keep_k + (1 if cls else 0)
    if y_kept is None:
        y_kept = torch.empty(B, n, C, dtype=torch.bfloat16, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(B, n, dtype=torch.int32, device=dev)
    if scores is None:
        scores = torch.empty(B, L, dtype=torch.float32, device=dev)
    st = lib().rs_block_forward_ex(_ptr(x), B, L, C, H, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                                   _ptr(gamma), _ptr(beta), int(keep_k), _dist(distance),
                                   0 if cls else RS_NO_CLS, _ptr(y_kept), _ptr(kept_idx),
                                   _ptr(scores), _stream(stream))
    _check(st, "rs_block_forward")
    return y_kept, kept_idx, scores


def rs_ln_stats(x2d: torch.Tensor, stats: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, C = x2d.shape
    if stats is None:
        stats = torch.empty(M, 2, dtype=torch.float32, device=x2d.device)
    _check(lib().rs_ln_stats(_ptr(x2d), M, C, _ptr(stats), _stream(stream)), "rs_ln_stats")
    return stats


def rs_ln_fc1_gelu(x2d: torch.Tensor, W1, b1, gamma, beta, hidden: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    M, C = x2d.shape
    H = W1.shape[0]
    if hidden is None:
        hidden = torch.empty(M, H, dtype=torch.bfloat16, device=x2d.device)
    st = lib().rs_ln_fc1_gelu(_ptr(x2d), M, C, H, _ptr(W1), _ptr(b1), _ptr(gamma), _ptr(beta),
                              _ptr(hidden), _stream(stream))
    _check(st, "rs_ln_fc1_gelu")
    return hidden


def rs_ln_fold(W1: torch.Tensor, b1, gamma, beta, Wg: Optional[torch.Tensor] = None,
               colG: Optional[torch.Tensor] = None, colC: Optional[torch.Tensor] = None,
               stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    H, C = W1.shape
    dev = W1.device
    if Wg is None:
        Wg = torch.empty(H, C, dtype=torch.bfloat16, device=dev)
    if colG is None:
        colG = torch.empty(H, dtype=torch.float32, device=dev)
    if colC is None:
        colC = torch.empty(H, dtype=torch.float32, device=dev)
    st = lib().rs_ln_fold(_ptr(W1), _ptr(b1), _ptr(gamma), _ptr(beta), C, H, _ptr(Wg), _ptr(colG),
                          _ptr(colC), _stream(stream))
    _check(st, "rs_ln_fold")
    return Wg, colG, colC


def rs_fc1_gelu_folded(x2d: torch.Tensor, stats, Wg, colG, colC,
                       hidden: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, C = x2d.shape
    H = Wg.shape[0]
    if hidden is None:
        hidden = torch.empty(M, H, dtype=torch.bfloat16, device=x2d.device)
    st = lib().rs_fc1_gelu_folded(_ptr(x2d), _ptr(stats), _ptr(Wg), _ptr(colG), _ptr(colC), M, C, H,
                                  _ptr(hidden), _stream(stream))
    _check(st, "rs_fc1_gelu_folded")
    return hidden


def rs_ln_fc1_gelu_staged(x2d: torch.Tensor, W1, b1, gamma, beta,
                          hidden: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    M, C = x2d.shape
    H = W1.shape[0]
    if hidden is None:
        hidden = torch.empty(M, H, dtype=torch.bfloat16, device=x2d.device)
    st = lib().rs_ln_fc1_gelu_staged(_ptr(x2d), M, C, H, _ptr(W1), _ptr(b1), _ptr(gamma),
                                     _ptr(beta), _ptr(hidden), _stream(stream))
    _check(st, "rs_ln_fc1_gelu_staged")
    return hidden


def rs_ln_fc1_gelu_noalloc(x2d: torch.Tensor, W1, b1, gamma, beta, hidden: torch.Tensor,
                           stream=None) -> torch.Tensor:
    """rs_ln_fc1_gelu with its scratch in the library's static device array (the caller
    provides ``hidden``; nothing is allocated)."""
    M, C = x2d.shape
    H = W1.shape[0]
    st = lib().rs_ln_fc1_gelu_noalloc(_ptr(x2d), M, C, H, _ptr(W1), _ptr(b1), _ptr(gamma),
                                      _ptr(beta), _ptr(hidden), _stream(stream))
    _check(st, "rs_ln_fc1_gelu_noalloc")
    return hidden


RS_FUSED_PARTIALS = 4


def rs_mlp_fused_supported(C: int, H: int) -> bool:
    return bool(lib().rs_mlp_fused_supported(int(C), int(H)))


def rs_mlp_fused(x2d: torch.Tensor, stats: torch.Tensor, Wg: torch.Tensor, colG: torch.Tensor,
                 colC: torch.Tensor, W2, b2, y: Optional[torch.Tensor] = None,
                 partials: Optional[torch.Tensor] = None, stream=None
                 ) -> Tuple[torch.Tensor, torch.Tensor]:
    """The fused MLP on LN statistics and folded weights: (y [M, C] bf16,
    partials [M, RS_FUSED_PARTIALS] fp32)."""
    M, C = x2d.shape
    H = Wg.shape[0]
    if y is None:
        y = torch.empty(M, C, dtype=torch.bfloat16, device=x2d.device)
    if partials is None:
        partials = torch.empty(M, RS_FUSED_PARTIALS, dtype=torch.float32, device=x2d.device)
    st = lib().rs_mlp_fused(_ptr(x2d), _ptr(stats), _ptr(Wg), _ptr(colG), _ptr(colC), M, C, H,
                            _ptr(W2), _ptr(b2), _ptr(y), _ptr(partials), _stream(stream))
    _check(st, "rs_mlp_fused")
    return y, partials


def rs_debug_fc1_skip_load(x2d: torch.Tensor, W1, b1, gamma, beta, hidden: torch.Tensor,
                           skip_kblock: int, timeout_us: int, stream=None) -> None:
    """Test hook: fc1 with one k-block load withheld (see include/rs.h)."""
    M, C = x2d.shape
    H = W1.shape[0]
    st = lib().rs_debug_fc1_skip_load(_ptr(x2d), M, C, H, _ptr(W1), _ptr(b1), _ptr(gamma),
                                      _ptr(beta), _ptr(hidden), int(skip_kblock), int(timeout_us),
                                      _stream(stream))
    _check(st, "rs_debug_fc1_skip_load")


def rs_gelu_apply(z: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty_like(z)
    _check(lib().rs_gelu_apply(_ptr(z), _ptr(out), z.numel(), _stream(stream)), "rs_gelu_apply")
    return out


def rs_num_partials(C: int, distance="l2") -> int:
    return int(lib().rs_num_partials_ex(int(C), _dist(distance)))


def rs_fc2_residual_shift(hidden: torch.Tensor, x2d: torch.Tensor, W2, b2,
                          y: Optional[torch.Tensor] = None, partials: Optional[torch.Tensor] = None,
                          stream=None, distance="l2") -> Tuple[torch.Tensor, torch.Tensor]:
    M, H = hidden.shape
    C = x2d.shape[1]
    if y is None:
        y = torch.empty(M, C, dtype=torch.bfloat16, device=x2d.device)
    if partials is None:
        partials = torch.empty(M, rs_num_partials(C, distance), dtype=torch.float32,
                               device=x2d.device)
    st = lib().rs_fc2_residual_shift_ex(_ptr(hidden), _ptr(x2d), M, C, H, _ptr(W2), _ptr(b2),
                                        _dist(distance), _ptr(y), _ptr(partials), _stream(stream))
    _check(st, "rs_fc2_residual_shift")
    return y, partials


def rs_select_topk(partials: torch.Tensor, B: int, L: int, keep_k: int,
                   scores: Optional[torch.Tensor] = None, kept_idx: Optional[torch.Tensor] = None,
                   stream=None, distance="l2", cls: bool = True) -> Tuple[torch.Tensor, torch.Tensor]:
    P = partials.shape[-1]
    dev = partials.device
    if scores is None:
        scores = torch.empty(B, L, dtype=torch.float32, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(B, keep_k + (1 if cls else 0), dtype=torch.int32, device=dev)
    st = lib().rs_select_topk_ex(_ptr(partials), P, B, L, int(keep_k), _dist(distance),
                                 0 if cls else RS_NO_CLS, _ptr(scores), _ptr(kept_idx),
                                 _stream(stream))
    _check(st, "rs_select_topk")
    return scores, kept_idx


def rs_select_gather(partials: torch.Tensor, y: torch.Tensor, keep_k: int,
                     scores: Optional[torch.Tensor] = None, kept_idx: Optional[torch.Tensor] = None,
                     y_kept: Optional[torch.Tensor] = None, stream=None, distance="l2",
                     cls: bool = True) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """partials [B*L, P] fp32, y [B, L, C] bf16 -> (scores, kept_idx, y_kept)."""
    B, L, C = y.shape
    P = partials.shape[-1]
    dev = y.device
    n = keep_k + (1 if cls else 0)
    if scores is None:
        scores = torch.empty(B, L, dtype=torch.float32, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(B, n, dtype=torch.int32, device=dev)
    if y_kept is None:
        y_kept = torch.empty(B, n, C, dtype=y.dtype, device=dev)
    st = lib().rs_select_gather_ex(_ptr(partials), P, _ptr(y), B, L, C, int(keep_k),
                                   _dist(distance), 0 if cls else RS_NO_CLS, _ptr(scores),
                                   _ptr(kept_idx), _ptr(y_kept), _stream(stream))
    _check(st, "rs_select_gather")
    return scores, kept_idx, y_kept


def rs_gather_rows(y: torch.Tensor, kept_idx: torch.Tensor, keep_k: int,
                   y_kept: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    B, L, C = y.shape
    if y_kept is None:
        y_kept = torch.empty(B, keep_k + 1, C, dtype=y.dtype, device=y.device)
    st = lib().rs_gather_rows(_ptr(y), B, L, C, _ptr(kept_idx), int(keep_k), _ptr(y_kept),
                              _stream(stream))
    _check(st, "rs_gather_rows")
    return y_kept


def rs_get_last_device_error(stream=None) -> int:
    return int(lib().rs_get_last_device_error(_stream(stream)))


def rs_release_workspace() -> None:
    lib().rs_release_workspace()


def rs_workspace_bytes(B: int, L: int, C: int, H: int) -> int:
    return int(lib().rs_workspace_bytes(B, L, C, H))


def rs_attn_core(qkv: torch.Tensor, heads: int, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """qkv [B, L, 3 * 64 heads] bf16 -> out [B, L, 64 heads] bf16: per sample and head,
    Softmax(Q K^T / 8) V."""
    B, L, C3 = qkv.shape
    C = 64 * heads
    if C3 != 3 * C:
        raise ValueError("qkv must be [B, L, 3 * 64 * heads]")
    if out is None:
        out = torch.empty(B, L, C, dtype=torch.bfloat16, device=qkv.device)
    _check(lib().rs_attn_core(_ptr(qkv), B, L, int(heads), _ptr(out), _stream(stream)),
           "rs_attn_core")
    return out


def rs_attn_sublayer(x: torch.Tensor, Wqkv, bqkv, Wo, bo, gamma, beta, heads: int,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x [B, L, C] bf16 -> x + SA(LN(x)) [B, L, C] bf16 (C = 64 heads)."""
    B, L, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check(lib().rs_attn_sublayer(_ptr(x), B, L, C, int(heads), _ptr(Wqkv), _ptr(bqkv), _ptr(Wo),
                                  _ptr(bo), _ptr(gamma), _ptr(beta), _ptr(out), _stream(stream)),
           "rs_attn_sublayer")
    return out


def rs_attn_forward(x: torch.Tensor, Wqkv, bqkv, Wo, bo, gamma, beta, heads: int, keep_k: int,
                    x_kept: Optional[torch.Tensor] = None,
                    kept_idx: Optional[torch.Tensor] = None,
                    scores: Optional[torch.Tensor] = None, stream=None, distance="l2",
                    cls: bool = True) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """The attention sublayer, then pruning by its representation shift:
    (x'_kept [B, n, C], kept_idx [B, n] int32, scores [B, L] fp32), n as in
    rs_block_forward."""
    B, L, C = x.shape
    dev = x.device
    n = keep_k + (1 if cls else 0)
    if x_kept is None:
        x_kept = torch.empty(B, n, C, dtype=torch.bfloat16, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(B, n, dtype=torch.int32, device=dev)
    if scores is None:
        scores = torch.empty(B, L, dtype=torch.float32, device=dev)
    st = lib().rs_attn_forward_ex(_ptr(x), B, L, C, int(heads), _ptr(Wqkv), _ptr(bqkv), _ptr(Wo),
                                  _ptr(bo), _ptr(gamma), _ptr(beta), int(keep_k), _dist(distance),
                                  0 if cls else RS_NO_CLS, _ptr(x_kept), _ptr(kept_idx),
                                  _ptr(scores), _stream(stream))
    _check(st, "rs_attn_forward")
    return x_kept, kept_idx, scores


def rs_mlp_forward(x: torch.Tensor, W1, b1, W2, b2, gamma, beta,
                   out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x [..., C] bf16 -> x + MLP(LN(x)) (no scoring, no pruning), same shape."""
    C = x.shape[-1]
    M = x.numel() // C
    H = W1.shape[0]
    if out is None:
        out = torch.empty_like(x)
    _check(lib().rs_mlp_forward(_ptr(x), M, C, H, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2),
                                _ptr(gamma), _ptr(beta), _ptr(out), _stream(stream)),
           "rs_mlp_forward")
    return out


ENCODER_WEIGHT_ORDER = ("Wqkv", "bqkv", "Wo", "bo", "gamma1", "beta1",
                        "W1", "b1", "W2", "b2", "gamma2", "beta2")


def rs_encoder_forward(x: torch.Tensor, layers, keep, heads: int,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x [B, L, C] bf16 through len(layers) encoder layers; `layers[l]` is a sequence
    of the 12 weight tensors in ENCODER_WEIGHT_ORDER, keep[l] the patch tokens kept
    after layer l (negative: no pruning). Returns [B, L_out, C]."""
    B, L, C = x.shape
    depth = len(layers)
    H = layers[0][6].shape[0]
    ptrs = (_vp * (12 * depth))(*[_ptr(t) for lw in layers for t in lw])
    kk = (_i * depth)(*[int(k) for k in keep])
    L_out = L
    for k in keep:
        if k >= 0:
            L_out = 1 + int(k)
    if out is None:
        out = torch.empty(B, L_out, C, dtype=torch.bfloat16, device=x.device)
    _check(lib().rs_encoder_forward(_ptr(x), B, L, C, H, int(heads), depth, ptrs, kk, _ptr(out),
                                    _stream(stream)), "rs_encoder_forward")
    return out


def rs_block_forward_block_shift(x_in: torch.Tensor, x: torch.Tensor, W1, b1, W2, b2, gamma,
                                 beta, keep_k: int, y_kept: Optional[torch.Tensor] = None,
                                 kept_idx: Optional[torch.Tensor] = None,
                                 scores: Optional[torch.Tensor] = None, stream=None,
                                 distance="l2", cls: bool = True):
    """rs_block_forward scored on the whole-block shift D(y, x_in): x_in [B, L, C] is the
    block input before the attention sublayer, x = x' its output."""
    B, L, C = x.shape
    H = W1.shape[0]
    dev = x.device
    n = keep_k + (1 if cls else 0)
    if y_kept is None:
        y_kept = torch.empty(B, n, C, dtype=torch.bfloat16, device=dev)
    if kept_idx is None:
        kept_idx = torch.empty(B, n, dtype=torch.int32, device=dev)
    if scores is None:
        scores = torch.empty(B, L, dtype=torch.float32, device=dev)
    st = lib().rs_block_forward_block_shift_ex(
        _ptr(x_in), _ptr(x), B, L, C, H, _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), _ptr(gamma),
        _ptr(beta), int(keep_k), _dist(distance), 0 if cls else RS_NO_CLS, _ptr(y_kept),
        _ptr(kept_idx), _ptr(scores), _stream(stream))
    _check(st, "rs_block_forward_block_shift")
    return y_kept, kept_idx, scores


def rs_debug_attn_skip_load(qkv: torch.Tensor, heads: int, out: torch.Tensor, skip_block: int,
                            timeout_us: int, stream=None) -> None:
    """Test hook: the attention core with one CTA's key-block loads withheld from
    `skip_block` on; its waits time out after `timeout_us` (see rs.h)."""
    B, L, _ = qkv.shape
    _check(lib().rs_debug_attn_skip_load(_ptr(qkv), B, L, int(heads), _ptr(out), int(skip_block),
                                         int(timeout_us), _stream(stream)),
           "rs_debug_attn_skip_load")
