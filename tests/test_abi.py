"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before launching anything (no GPU)."""
import ctypes
import os
import re

import pytest

import free_vit_token_b200.rs as rs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned fake device address: never dereferenced on these paths
MIS = 0x10002   # misaligned fake address


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rs.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rs_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "rs_block_forward" in names and len(names) >= 10
    lib = rs.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rs.SIGNATURES), "binding and header disagree"


def test_status_strings():
    for code in range(8):
        assert rs.status_string(code).startswith("RS_")
    assert "unknown" in rs.status_string(99)


def test_num_partials_and_workspace():
    assert rs.rs_num_partials(384) == 4      # two 192-wide tiles, two column groups each
    assert rs.rs_num_partials(768) == 6
    assert rs.rs_num_partials(1024) == 8
    assert rs.rs_num_partials(192) == 2
    assert rs.rs_num_partials(100) == 0
    wb = rs.rs_workspace_bytes(256, 197, 384, 1536)
    M = 256 * 197
    assert wb >= M * 1536 * 2 + M * 384 * 2 + M * 8 + M * 4 * 4
    assert rs.rs_workspace_bytes(1, 1, 65, 64) == 0


def _fwd(x=FAKE, B=2, L=197, C=192, H=768, w=FAKE, keep_k=137, out=FAKE, idx=FAKE, sc=FAKE):
    return rs.lib().rs_block_forward(x, B, L, C, H, w, w, w, w, w, w, keep_k, out, idx, sc, None)


def test_block_forward_argument_errors():
    assert _fwd(B=0) == rs.RS_OK                  # empty batch: nothing to do
    assert _fwd(B=0, x=None, out=None) == rs.RS_OK
    assert _fwd(x=None) == rs.RS_ERR_NULL
    assert _fwd(w=None) == rs.RS_ERR_NULL
    assert _fwd(idx=None) == rs.RS_ERR_NULL
    assert _fwd(B=-1) == rs.RS_ERR_SHAPE
    assert _fwd(L=0) == rs.RS_ERR_SHAPE
    assert _fwd(L=16385, keep_k=1) == rs.RS_ERR_SHAPE
    assert _fwd(C=200) == rs.RS_ERR_SHAPE
    assert _fwd(C=4096) == rs.RS_ERR_SHAPE
    assert _fwd(H=100) == rs.RS_ERR_SHAPE
    assert _fwd(B=1 << 20, C=2048, H=2048, L=1024) == rs.RS_ERR_SHAPE
    assert _fwd(keep_k=-1) == rs.RS_ERR_KEEP_K
    assert _fwd(keep_k=197) == rs.RS_ERR_KEEP_K
    assert _fwd(x=MIS) == rs.RS_ERR_ALIGN
    assert _fwd(out=MIS) == rs.RS_ERR_ALIGN
    assert _fwd(idx=FAKE + 1) == rs.RS_ERR_ALIGN


def test_step_entry_points_argument_errors():
    L = rs.lib()
    assert L.rs_ln_stats(None, 10, 192, FAKE, None) == rs.RS_ERR_NULL
    assert L.rs_ln_stats(FAKE, 10, 100, FAKE, None) == rs.RS_ERR_SHAPE
    assert L.rs_ln_stats(FAKE, 0, 192, FAKE, None) == rs.RS_OK
    assert L.rs_ln_fc1_gelu(FAKE, 10, 192, 770, FAKE, FAKE, FAKE, FAKE, FAKE, None) == rs.RS_ERR_SHAPE
    assert L.rs_ln_fc1_gelu(FAKE, 10, 192, 768, None, FAKE, FAKE, FAKE, FAKE, None) == rs.RS_ERR_NULL
    assert L.rs_ln_fc1_gelu(MIS, 10, 192, 768, FAKE, FAKE, FAKE, FAKE, FAKE, None) == rs.RS_ERR_ALIGN
    assert L.rs_fc2_residual_shift(FAKE, FAKE, 10, 192, 768, FAKE, FAKE, FAKE, None, None) == rs.RS_ERR_NULL
    assert L.rs_select_topk(FAKE, 0, 2, 10, 3, FAKE, FAKE, None) == rs.RS_ERR_SHAPE
    assert L.rs_select_topk(FAKE, 4, 2, 10, 10, FAKE, FAKE, None) == rs.RS_ERR_KEEP_K
    assert L.rs_select_topk(FAKE, 4, 0, 10, 3, None, None, None) == rs.RS_OK
    assert L.rs_select_topk(FAKE, 4, 2, 10, 3, FAKE, FAKE + 2, None) == rs.RS_ERR_ALIGN
    assert L.rs_gather_rows(FAKE, 2, 10, 192, FAKE, 10, FAKE, None) == rs.RS_ERR_KEEP_K
    assert L.rs_gather_rows(FAKE, 2, 10, 192, None, 3, FAKE, None) == rs.RS_ERR_NULL


def test_extended_entry_points_argument_errors():
    L = rs.lib()
    NO_CLS, COS, L1_ = rs.RS_NO_CLS, rs.RS_DIST_COSINE, rs.RS_DIST_L1
    assert L.rs_num_partials_ex(384, COS) == 3 * L.rs_num_partials(384) == 12
    assert L.rs_num_partials_ex(768, L1_) == L.rs_num_partials(768)
    assert L.rs_num_partials_ex(384, 3) == 0
    sel = lambda np_, B, Lq, k, d, f, kept=FAKE: L.rs_select_topk_ex(FAKE, np_, B, Lq, k, d, f,
                                                                      FAKE, kept, None)
    assert sel(6, 2, 10, 3, 3, 0) == rs.RS_ERR_SHAPE           # unknown distance
    assert sel(6, 2, 10, 3, 0, 2) == rs.RS_ERR_SHAPE           # unknown flag
    assert sel(4, 2, 10, 3, COS, 0) == rs.RS_ERR_SHAPE         # cosine partials are triples
    assert sel(66, 2, 10, 3, COS, 0) == rs.RS_ERR_SHAPE        # more than 64 partials
    assert sel(6, 2, 10, 10, 0, 0) == rs.RS_ERR_KEEP_K         # keep_k = L needs no CLS
    assert sel(6, 2, 10, 11, 0, NO_CLS) == rs.RS_ERR_KEEP_K
    assert sel(6, 0, 10, 10, 0, NO_CLS) == rs.RS_OK            # empty batch
    assert sel(6, 2, 10, 3, COS, NO_CLS, kept=FAKE + 2) == rs.RS_ERR_ALIGN
    fwd = lambda k, d, f: L.rs_block_forward_ex(FAKE, 2, 10, 192, 768, FAKE, FAKE, FAKE, FAKE,
                                                FAKE, FAKE, k, d, f, FAKE, FAKE, FAKE, None)
    assert fwd(3, 5, 0) == rs.RS_ERR_SHAPE
    assert fwd(3, 0, 4) == rs.RS_ERR_SHAPE
    assert fwd(10, 0, 0) == rs.RS_ERR_KEEP_K
    assert fwd(-1, 0, NO_CLS) == rs.RS_ERR_KEEP_K
    assert L.rs_fc2_residual_shift_ex(FAKE, FAKE, 10, 192, 768, FAKE, FAKE, 9, FAKE, FAKE,
                                      None) == rs.RS_ERR_SHAPE
    assert L.rs_select_gather_ex(FAKE, 6, FAKE, 2, 10, 192, 3, COS, 0, FAKE, FAKE, MIS,
                                 None) == rs.RS_ERR_ALIGN


def test_attention_entry_points_argument_errors():
    lib = rs.lib()
    w = FAKE

    def sub(x=FAKE, B=2, L=197, C=384, heads=6, wt=w, out=FAKE):
        return lib.rs_attn_sublayer(x, B, L, C, heads, wt, wt, wt, wt, wt, wt, out, None)

    def fwd(B=2, L=197, C=384, heads=6, k=137, dist=0, flags=0, out=FAKE, idx=FAKE, sc=FAKE):
        return lib.rs_attn_forward_ex(FAKE, B, L, C, heads, w, w, w, w, w, w, k, dist, flags,
                                      out, idx, sc, None)

    assert lib.rs_attn_core(FAKE, 0, 7, 2, FAKE, None) == rs.RS_OK     # empty batch
    assert lib.rs_attn_core(None, 1, 7, 2, FAKE, None) == rs.RS_ERR_NULL
    assert lib.rs_attn_core(FAKE, 1, 7, 2, None, None) == rs.RS_ERR_NULL
    assert lib.rs_attn_core(MIS, 1, 7, 2, FAKE, None) == rs.RS_ERR_ALIGN
    assert lib.rs_attn_core(FAKE, 1, 0, 2, FAKE, None) == rs.RS_ERR_SHAPE
    assert lib.rs_attn_core(FAKE, 1, 7, 0, FAKE, None) == rs.RS_ERR_SHAPE
    assert lib.rs_attn_core(FAKE, 1, 7, 33, FAKE, None) == rs.RS_ERR_SHAPE  # 64 * 33 > RS_MAX_C
    assert lib.rs_attn_core(FAKE, 1, 16385, 2, FAKE, None) == rs.RS_ERR_SHAPE
    assert sub(B=0) == rs.RS_OK
    assert sub(C=384, heads=4) == rs.RS_ERR_SHAPE       # heads of width 64 only
    assert sub(C=96, heads=1) == rs.RS_ERR_SHAPE
    assert sub(x=None) == rs.RS_ERR_NULL
    assert sub(wt=None) == rs.RS_ERR_NULL
    assert sub(out=None) == rs.RS_ERR_NULL
    assert sub(out=MIS) == rs.RS_ERR_ALIGN
    assert sub(x=MIS) == rs.RS_ERR_ALIGN
    assert fwd(B=0) == rs.RS_OK
    assert fwd(k=197) == rs.RS_ERR_KEEP_K               # CLS kept: at most L - 1
    assert fwd(k=198, flags=rs.RS_NO_CLS) == rs.RS_ERR_KEEP_K
    assert fwd(k=-1) == rs.RS_ERR_KEEP_K
    assert fwd(dist=3) == rs.RS_ERR_SHAPE
    assert fwd(flags=2) == rs.RS_ERR_SHAPE
    assert fwd(sc=None) == rs.RS_ERR_NULL
    assert fwd(idx=None) == rs.RS_ERR_NULL
    assert fwd(out=MIS) == rs.RS_ERR_ALIGN
    assert fwd(heads=5) == rs.RS_ERR_SHAPE


def test_encoder_and_mlp_entry_points_argument_errors():
    lib = rs.lib()
    depth = 3
    good = (ctypes.c_void_p * (12 * depth))(*([FAKE] * (12 * depth)))
    holes = (ctypes.c_void_p * (12 * depth))(*([FAKE] * (12 * depth - 1) + [None]))
    mis = (ctypes.c_void_p * (12 * depth))(*([FAKE] * 5 + [MIS] + [FAKE] * (12 * depth - 6)))

    def keep(*k):
        return (ctypes.c_int * depth)(*k)

    def enc(x=FAKE, B=2, L=197, C=384, H=1536, heads=6, w=good, k=None, out=FAKE, d=depth):
        return lib.rs_encoder_forward(x, B, L, C, H, heads, d, w,
                                      k if k is not None else keep(-1, 157, -1), out, None)

    assert enc(B=0) == rs.RS_OK
    assert enc(x=None) == rs.RS_ERR_NULL
    assert enc(out=None) == rs.RS_ERR_NULL
    assert enc(w=holes) == rs.RS_ERR_NULL
    assert enc(w=mis) == rs.RS_ERR_ALIGN
    assert enc(heads=5) == rs.RS_ERR_SHAPE
    assert enc(H=100) == rs.RS_ERR_SHAPE
    assert enc(d=0) == rs.RS_ERR_SHAPE
    assert enc(k=keep(-1, 197, -1)) == rs.RS_ERR_KEEP_K        # more than L - 1 patches
    assert enc(k=keep(100, 101, -1)) == rs.RS_ERR_KEEP_K       # later layer keeps more
    assert lib.rs_mlp_forward(FAKE, 0, 384, 1536, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              None) == rs.RS_OK
    assert lib.rs_mlp_forward(FAKE, 10, 384, 1536, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                              None) == rs.RS_ERR_NULL
    assert lib.rs_mlp_forward(FAKE, 10, 100, 1536, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              None) == rs.RS_ERR_SHAPE
    assert lib.rs_mlp_forward(MIS, 10, 384, 1536, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                              None) == rs.RS_ERR_ALIGN


def test_fused_mlp_entry_point_argument_errors():
    lib = rs.lib()

    def f(x=FAKE, st=FAKE, M=300, C=384, H=1536, y=FAKE, part=FAKE):
        return lib.rs_mlp_fused(x, st, FAKE, FAKE, FAKE, M, C, H, FAKE, FAKE, y, part, None)

    assert lib.rs_mlp_fused_supported(384, 1536) == 1
    assert lib.rs_mlp_fused_supported(64, 128) == 1
    assert lib.rs_mlp_fused_supported(448, 1792) == 0    # wider than TMEM holds with T1
    assert lib.rs_mlp_fused_supported(384, 1600) == 0    # hidden width not in 128 chunks
    assert f(M=0) == rs.RS_OK
    assert f(C=448, H=1792) == rs.RS_ERR_SHAPE
    assert f(C=100) == rs.RS_ERR_SHAPE
    assert f(x=None) == rs.RS_ERR_NULL
    assert f(part=None) == rs.RS_ERR_NULL
    assert f(x=MIS) == rs.RS_ERR_ALIGN
    assert f(st=FAKE + 4) == rs.RS_ERR_ALIGN
    assert f(part=FAKE + 2) == rs.RS_ERR_ALIGN


def test_block_shift_entry_point_argument_errors():
    lib = rs.lib()
    w = FAKE

    def f(x_in=FAKE, x=FAKE, B=2, L=197, C=192, H=768, k=137, dist=0, flags=0, out=FAKE,
          idx=FAKE, sc=FAKE):
        return lib.rs_block_forward_block_shift_ex(x_in, x, B, L, C, H, w, w, w, w, w, w, k,
                                                   dist, flags, out, idx, sc, None)

    assert f(B=0) == rs.RS_OK
    assert f(x_in=None) == rs.RS_ERR_NULL
    assert f(x_in=MIS) == rs.RS_ERR_ALIGN
    assert f(x=None) == rs.RS_ERR_NULL
    assert f(k=197) == rs.RS_ERR_KEEP_K
    assert f(dist=7) == rs.RS_ERR_SHAPE
    assert f(C=100) == rs.RS_ERR_SHAPE
    assert f(sc=None) == rs.RS_ERR_NULL


def test_library_has_no_torch_or_libcuda_link_dependency():
    out = os.popen(f"ldd {rs.LIB_PATH}").read()
    assert "libtorch" not in out and "libc10" not in out
