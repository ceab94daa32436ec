// rs_api.cu -- the C ABI of librs.so (declared and documented in include/rs.h):
// argument validation, the per-device workspace, TMA tensor maps and the launch
// sequence of the pruned-MLP block of "Representation Shift: Unifying Token
// Compression with FlashAttention" (§3.3 Eq. (6), §3.2 Eq. (4), §3.1 pruning).
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "rs.h"
#include "rs_internal.h"

namespace rs {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A 2-D bf16 tensor map (layout and swizzle choice as declared in rs_internal.h).
int make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows,
              uint32_t box_inner) {
  auto fn = encode_fn();
  if (fn == nullptr) return RS_ERR_CUDA;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = box_inner == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : box_inner == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RS_OK : RS_ERR_CUDA;
}

}  // namespace rs

namespace {

constexpr int kMaxDevices = 64;
using rs::encode_fn;
using rs::make_tmap;

struct DevState {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  void* act = nullptr;  // rs_encoder_forward: activations between layers
  size_t act_bytes = 0;
  int* err = nullptr;  // device status flag (one int)
  int num_sms = 0;
};

std::mutex g_mu;
DevState g_dev[kMaxDevices];

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace: the fc1 part (LN statistics and the folded weights) first, then
// the block's intermediates.
struct WsLayout {
  size_t stats, wg, colg, colc, fc1_total, hidden, y, partials, total;
};

WsLayout ws_layout(int64_t M, int C, int H) {
  WsLayout w{};
  size_t off = 0;
  w.stats = off;
  off = align_up(off + static_cast<size_t>(M) * 8, 1024);
  w.wg = off;
  off = align_up(off + static_cast<size_t>(H) * C * 2, 1024);
  w.colg = off;
  off = align_up(off + static_cast<size_t>(H) * 4, 1024);
  w.colc = off;
  off = align_up(off + static_cast<size_t>(H) * 4, 1024);
  w.fc1_total = off;
  w.hidden = off;
  off = align_up(off + static_cast<size_t>(M) * H * 2, 1024);
  w.y = off;
  off = align_up(off + static_cast<size_t>(M) * C * 2, 1024);
  w.partials = off;  // room for the cosine distance's three partials per column group
  off = align_up(off + static_cast<size_t>(M) * rs::dist_partials(rs::kDistCos) *
                           (rs::kFc2PartialsPerTile * C / rs::fc2_block_n(C)) * 4,
                 1024);
  w.total = off;
  return w;
}

// Caller holds g_mu.
int dev_state(DevState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RS_ERR_CUDA;
  DevState& st = g_dev[dev];
  if (st.err == nullptr) {
    if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return RS_ERR_CUDA;
    int* e = nullptr;
    if (cudaMalloc(&e, 256) != cudaSuccess) return RS_ERR_NO_MEM;
    if (cudaMemset(e, 0, 256) != cudaSuccess) return RS_ERR_CUDA;
    st.err = e;
  }
  *out = &st;
  return RS_OK;
}

// Caller holds g_mu. Grows a cached buffer in stream order on `s`: the old one is
// released with cudaFreeAsync and the new one taken with cudaMallocAsync, so no
// call synchronises the device. The buffer is shared by every call on the device
// (calls on different streams must be ordered by the caller). It cannot grow while
// `s` is being captured into a graph: an allocation made during capture would
// belong to the graph, so the call fails with RS_ERR_NO_MEM and the caller makes
// one call at the largest size before capturing.
int grow_buffer(void** buf, size_t* cur, size_t bytes, cudaStream_t s) {
  if (*cur >= bytes) return RS_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  if (cs != cudaStreamCaptureStatusNone) return RS_ERR_NO_MEM;
  if (*buf != nullptr) {
    if (cudaFreeAsync(*buf, s) != cudaSuccess) {
      cudaGetLastError();
      return RS_ERR_CUDA;
    }
    *buf = nullptr;
    *cur = 0;
  }
  if (cudaMallocAsync(buf, bytes, s) != cudaSuccess) {
    cudaGetLastError();
    *buf = nullptr;
    return RS_ERR_NO_MEM;
  }
  *cur = bytes;
  return RS_OK;
}
int ensure_ws(DevState& st, size_t bytes, cudaStream_t s) {
  return grow_buffer(&st.ws, &st.ws_bytes, bytes, s);
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al8(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 7u) == 0; }
bool al4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_width(int C) {
  return (C < 64 || C > RS_MAX_C || C % 64 != 0) ? RS_ERR_SHAPE : RS_OK;
}
int check_hidden(int H) {
  return (H < 64 || H > RS_MAX_H || H % 64 != 0) ? RS_ERR_SHAPE : RS_OK;
}
int check_rows(int64_t M, int C, int H) {
  if (M < 0) return RS_ERR_SHAPE;
  const int64_t w = C > H ? C : H;
  return (M * w >= (static_cast<int64_t>(1) << 31)) ? RS_ERR_SHAPE : RS_OK;
}

#define RS_TRY(expr)              \
  do {                            \
    const int _s = (expr);        \
    if (_s != RS_OK) return _s;   \
  } while (0)
#define RS_CUDA(expr)                                       \
  do {                                                      \
    if ((expr) != cudaSuccess) {                            \
      cudaGetLastError();                                   \
      return RS_ERR_CUDA;                                   \
    }                                                       \
  } while (0)

// LN statistics (and, for the folded LN, the weight fold in the same launch),
// then fc1 with the LayerNorm folded into the GEMM (default) or staged into the
// A operand by LN warps (staged = true). `ws` holds the fc1 part of the
// workspace layout for these sizes. The first launch follows the stream's
// previous work normally; the GEMM is a programmatic dependent launch.
int run_fc1(DevState& st, const void* x, int M, int C, int H, const void* W1, const void* b1,
            const void* gamma, const void* beta, uint8_t* ws, const WsLayout& w, void* hidden,
            bool staged, cudaStream_t s, bool linear = false) {
  float* stats = reinterpret_cast<float*>(ws + w.stats);
  const int bn = rs::fc1_block_n(H);
  const bool pair = rs::gemm_pair(M, C, staged);
  rs::MlpParams p{};
  p.M = M;
  p.N = H;
  p.K = C;
  p.n_blocks = H / bn;
  p.num_tiles = rs::gemm_num_tiles(M, p.n_blocks, pair);
  p.stats = reinterpret_cast<const float2*>(stats);
  p.out = static_cast<__nv_bfloat16*>(hidden);
  p.err = st.err;
  p.timeout_ns = rs::kDefaultTimeoutNs;
  p.debug_skip_kb = -1;
  p.linear = linear ? 1 : 0;
  const void* wB = W1;
  if (staged) {
    RS_CUDA(rs::launch_ln_stats(x, M, C, stats, st.num_sms, s));
    p.ln_gamma = static_cast<const __nv_bfloat16*>(gamma);
    p.ln_beta = static_cast<const __nv_bfloat16*>(beta);
    p.bias = static_cast<const __nv_bfloat16*>(b1);
  } else {
    void* wg = ws + w.wg;
    float* colg = reinterpret_cast<float*>(ws + w.colg);
    float* colc = reinterpret_cast<float*>(ws + w.colc);
    RS_CUDA(rs::launch_ln_prep(x, M, C, stats, W1, gamma, beta, b1, H, wg, colg, colc, st.num_sms,
                               s));
    p.colG = colg;
    p.colC = colc;
    wB = wg;
  }
  CUtensorMap tmX, tmW, tmHid;
  RS_TRY(make_tmap(&tmX, x, C, M, 128));
  RS_TRY(make_tmap(&tmW, wB, C, H, rs::gemm_b_box_rows(bn, pair)));
  RS_TRY(make_tmap(&tmHid, hidden, H, M, rs::kEpiBoxRows, rs::fc1_out_box_cols(H, C, staged)));
  RS_CUDA(rs::launch_fc1(tmX, tmW, tmHid, p, bn, staged, pair, st.num_sms, s, /*pdl=*/true));
  return RS_OK;
}

int run_fc2(DevState& st, const void* hidden, const void* x, int M, int C, int H, const void* W2,
            const void* b2, void* y, float* partials, int dist, cudaStream_t s, bool pdl = false,
            const void* shift_ref = nullptr) {
  const int bn = rs::fc2_block_n(C);
  const bool pair = rs::gemm_pair(M, H, false);
  CUtensorMap tmH, tmW, tmY;
  RS_TRY(make_tmap(&tmH, hidden, H, M, 128));
  RS_TRY(make_tmap(&tmW, W2, H, C, rs::gemm_b_box_rows(bn, pair)));
  RS_TRY(make_tmap(&tmY, y, C, M, rs::kEpiBoxRows, rs::fc2_out_box_cols(C)));
  rs::MlpParams p{};
  p.M = M;
  p.N = C;
  p.K = H;
  p.n_blocks = C / bn;
  p.num_tiles = rs::gemm_num_tiles(M, p.n_blocks, pair);
  p.bias = static_cast<const __nv_bfloat16*>(b2);
  p.out = static_cast<__nv_bfloat16*>(y);
  p.resid = static_cast<const __nv_bfloat16*>(x);
  p.partials = partials;
  p.dist = dist;
  p.shift_ref = static_cast<const __nv_bfloat16*>(shift_ref);
  p.num_partials = rs::dist_partials(dist) * rs::kFc2PartialsPerTile * p.n_blocks;
  p.err = st.err;
  p.timeout_ns = rs::kDefaultTimeoutNs;
  p.debug_skip_kb = -1;
  RS_CUDA(rs::launch_fc2(tmH, tmW, tmY, p, bn, pair, st.num_sms, s, pdl));
  return RS_OK;
}

// The fused MLP (rs_fused.cu) on LN statistics and folded weights already in place.
int run_fused_step(DevState& st, const void* x, const float* stats, const void* wg,
                   const float* colg, const float* colc, int M, int C, int H, const void* W2,
                   const void* b2, void* y, float* partials, cudaStream_t s, bool pdl) {
  CUtensorMap tmX, tmWg, tmW2, tmY;
  RS_TRY(make_tmap(&tmX, x, C, M, 128));
  RS_TRY(make_tmap(&tmWg, wg, C, H, 128));
  RS_TRY(make_tmap(&tmW2, W2, H, C, rs::fused_w2_rows(C)));
  RS_TRY(make_tmap(&tmY, y, C, M, rs::kEpiBoxRows, 16));
  rs::FusedParams p{};
  p.M = M;
  p.C = C;
  p.H = H;
  p.num_m = (M + 127) / 128;
  p.stats = reinterpret_cast<const float2*>(stats);
  p.colG = colg;
  p.colC = colc;
  p.b2 = static_cast<const __nv_bfloat16*>(b2);
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.partials = partials;
  p.err = st.err;
  p.timeout_ns = rs::kDefaultTimeoutNs;
  RS_CUDA(rs::launch_mlp_fused(tmX, tmWg, tmW2, tmY, p, st.num_sms, s, pdl));
  return RS_OK;
}

// The distance (RS_DIST_*) and the flags (RS_NO_CLS) of an extended entry point.
int check_mode(int distance, int flags) {
  if (distance != RS_DIST_L2 && distance != RS_DIST_L1 && distance != RS_DIST_COSINE)
    return RS_ERR_SHAPE;
  if ((flags & ~RS_NO_CLS) != 0) return RS_ERR_SHAPE;
  return RS_OK;
}
// keep_k: 0..L-1 patch tokens with a CLS token, 0..L tokens without.
int check_keep(int keep_k, int L, int flags) {
  const int max_k = (flags & RS_NO_CLS) ? L : L - 1;
  return (keep_k < 0 || keep_k > max_k) ? RS_ERR_KEEP_K : RS_OK;
}
// Partials per row: 1..64, and whole triples for the cosine distance.
int check_partials(int num_partials, int distance) {
  if (num_partials < 1 || num_partials > 64) return RS_ERR_SHAPE;
  if (distance == RS_DIST_COSINE && num_partials % 3 != 0) return RS_ERR_SHAPE;
  return RS_OK;
}

// ---------------------------------------------------------------- attention sublayer
// Workspace of the attention sublayer: the QKV projection's LN statistics and
// folded weights (the fc1 fields of WsLayout), the projection [M, 3C] (`hidden`),
// x' [M, C] (`y`, pruning variant), the shift partials, and the attention
// output [M, C] at `o`.
struct AttnWs {
  WsLayout w;
  size_t o;
};
AttnWs attn_ws_layout(int64_t M, int C) {
  AttnWs a{};
  WsLayout& w = a.w;
  size_t off = 0;
  w.stats = off;
  off = align_up(off + static_cast<size_t>(M) * 8, 1024);
  w.wg = off;
  off = align_up(off + static_cast<size_t>(3 * C) * C * 2, 1024);
  w.colg = off;
  off = align_up(off + static_cast<size_t>(3 * C) * 4, 1024);
  w.colc = off;
  off = align_up(off + static_cast<size_t>(3 * C) * 4, 1024);
  w.fc1_total = off;
  w.hidden = off;
  off = align_up(off + static_cast<size_t>(M) * 3 * C * 2, 1024);
  w.y = off;
  off = align_up(off + static_cast<size_t>(M) * C * 2, 1024);
  w.partials = off;
  off = align_up(off + static_cast<size_t>(M) * rs::dist_partials(rs::kDistCos) *
                           (rs::kFc2PartialsPerTile * C / rs::fc2_block_n(C)) * 4,
                 1024);
  a.o = off;
  off = align_up(off + static_cast<size_t>(M) * C * 2, 1024);
  w.total = off;
  return a;
}

// The QKV projection [B*L, 3C] as a [B][L][3C] tensor with {64, box_rows, 1} boxes.
int make_tmap_qkv(CUtensorMap* m, const void* qkv, int B, int L, int C, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return RS_ERR_CUDA;
  const cuuint64_t row = static_cast<cuuint64_t>(3 * C) * 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(3 * C), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {row, row * static_cast<cuuint64_t>(L)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qkv), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RS_OK : RS_ERR_CUDA;
}

// Heads of width 64: C = 64 heads, within the library's width limit.
int check_heads(int C, int heads) {
  if (heads < 1 || C != 64 * heads) return RS_ERR_SHAPE;
  return check_width(C);
}

int run_attn_core(DevState& st, const void* qkv, int B, int L, int C, int heads, void* out,
                  cudaStream_t s, bool pdl, int debug_skip_block = -1,
                  unsigned long long timeout_ns = rs::kDefaultTimeoutNs) {
  CUtensorMap tmQ, tmKV;
  RS_TRY(make_tmap_qkv(&tmQ, qkv, B, L, C, rs::attn_q_box_rows()));
  RS_TRY(make_tmap_qkv(&tmKV, qkv, B, L, C, rs::attn_kv_box_rows()));
  rs::AttnParams p{};
  p.B = B;
  p.L = L;
  p.C = C;
  p.heads = heads;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = st.err;
  p.timeout_ns = timeout_ns;
  p.debug_skip_block = debug_skip_block;
  RS_CUDA(rs::launch_attn(tmQ, tmKV, p, s, pdl));
  return RS_OK;
}

// x_out = x + SA(LN(x)) Wo^T + bo, and the shift partials of D(SA(LN(x)), x):
// LN prep + QKV projection (the folded-LN GEMM without activation), the
// attention core, the output projection (the fc2 GEMM with K = C).
int run_attn_sublayer(DevState& st, const void* x, int B, int L, int C, int heads,
                      const void* Wqkv, const void* bqkv, const void* Wo, const void* bo,
                      const void* gamma, const void* beta, void* x_out, int distance,
                      cudaStream_t s, uint8_t** ws_out, WsLayout* w_out) {
  const int64_t M64 = static_cast<int64_t>(B) * L;
  const int M = static_cast<int>(M64);
  const AttnWs aw = attn_ws_layout(M64, C);
  const WsLayout& w = aw.w;
  RS_TRY(ensure_ws(st, w.total, s));
  uint8_t* ws = static_cast<uint8_t*>(st.ws);
  void* qkv = ws + w.hidden;
  void* attn_o = ws + aw.o;
  float* partials = reinterpret_cast<float*>(ws + w.partials);
  RS_TRY(run_fc1(st, x, M, C, 3 * C, Wqkv, bqkv, gamma, beta, ws, w, qkv, false, s,
                 /*linear=*/true));
  RS_TRY(run_attn_core(st, qkv, B, L, C, heads, attn_o, s, /*pdl=*/true));
  RS_TRY(run_fc2(st, attn_o, x, M, C, C, Wo, bo, x_out ? x_out : ws + w.y, partials, distance, s,
                 /*pdl=*/true));
  if (ws_out) *ws_out = ws;
  if (w_out) *w_out = w;
  return RS_OK;
}

// The pruned MLP block (rs_block_forward_ex's launches) on validated arguments.
int run_block(DevState& st, const void* x, int B, int L, int C, int H, const void* W1,
              const void* b1, const void* W2, const void* b2, const void* gamma,
              const void* beta, int keep_k, int distance, int flags, void* y_kept,
              int32_t* kept_idx, float* scores, cudaStream_t s,
              const void* shift_ref = nullptr) {
  const int M = B * L;
  const WsLayout w = ws_layout(M, C, H);
  RS_TRY(ensure_ws(st, w.total, s));
  uint8_t* ws = static_cast<uint8_t*>(st.ws);
  void* hidden = ws + w.hidden;
  void* y = ws + w.y;
  float* partials = reinterpret_cast<float*>(ws + w.partials);
  const int np =
      rs::dist_partials(distance) * rs::kFc2PartialsPerTile * C / rs::fc2_block_n(C);
  RS_TRY(run_fc1(st, x, M, C, H, W1, b1, gamma, beta, ws, w, hidden, false, s));
  RS_TRY(run_fc2(st, hidden, x, M, C, H, W2, b2, y, partials, distance, s, /*pdl=*/true,
                 shift_ref));
  RS_CUDA(rs::launch_select_gather(partials, np, y, B, L, C, keep_k, distance,
                                   !(flags & RS_NO_CLS), scores, kept_idx, y_kept, st.num_sms, s,
                                   /*pdl=*/true));
  return RS_OK;
}

// The non-pruning MLP sublayer (rs_mlp_forward's launches) on validated arguments.
int run_mlp(DevState& st, const void* x, int M, int C, int H, const void* W1, const void* b1,
            const void* W2, const void* b2, const void* gamma, const void* beta, void* y,
            cudaStream_t s) {
  const WsLayout w = ws_layout(M, C, H);
  RS_TRY(ensure_ws(st, w.total, s));
  uint8_t* ws = static_cast<uint8_t*>(st.ws);
  void* hidden = ws + w.hidden;
  RS_TRY(run_fc1(st, x, M, C, H, W1, b1, gamma, beta, ws, w, hidden, false, s));
  RS_TRY(run_fc2(st, hidden, x, M, C, H, W2, b2, y, reinterpret_cast<float*>(ws + w.partials),
                 RS_DIST_L2, s, /*pdl=*/true));
  return RS_OK;
}

// Caller holds g_mu; grows the encoder's activation buffer (as the workspace).
int ensure_act(DevState& st, size_t bytes, cudaStream_t s) {
  return grow_buffer(&st.act, &st.act_bytes, bytes, s);
}

int check_attn_args(const void* x, int B, int L, int C, int heads, const void* Wqkv,
                    const void* bqkv, const void* Wo, const void* bo, const void* gamma,
                    const void* beta) {
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_heads(C, heads));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, 3 * C));
  if (B == 0) return RS_OK;
  if (!x || !Wqkv || !bqkv || !Wo || !bo || !gamma || !beta) return RS_ERR_NULL;
  if (!al16(x) || !al16(Wqkv) || !al16(bqkv) || !al16(Wo) || !al16(bo) || !al16(gamma) ||
      !al16(beta))
    return RS_ERR_ALIGN;
  return RS_OK;
}

}  // namespace

extern "C" {

const char* rs_status_string(int status) {
  switch (status) {
    case RS_OK: return "RS_OK";
    case RS_ERR_NULL: return "RS_ERR_NULL: a required pointer is NULL";
    case RS_ERR_SHAPE: return "RS_ERR_SHAPE: B, L, C or H outside the supported limits";
    case RS_ERR_KEEP_K:
      return "RS_ERR_KEEP_K: keep_k outside 0..L-1 (0..L without a CLS token)";
    case RS_ERR_ALIGN: return "RS_ERR_ALIGN: a pointer is not suitably aligned";
    case RS_ERR_CUDA: return "RS_ERR_CUDA: the CUDA runtime or driver reported an error";
    case RS_ERR_DEVICE_TIMEOUT: return "RS_ERR_DEVICE_TIMEOUT: a kernel pipeline wait timed out";
    case RS_ERR_NO_MEM:
      return "RS_ERR_NO_MEM: workspace allocation failed (or growth needed during stream capture)";
    default: return "unknown rs_status";
  }
}

int rs_num_partials_ex(int C, int distance) {
  if (check_width(C) != RS_OK || check_mode(distance, 0) != RS_OK) return 0;
  return rs::dist_partials(distance) * rs::kFc2PartialsPerTile * C / rs::fc2_block_n(C);
}
int rs_num_partials(int C) { return rs_num_partials_ex(C, RS_DIST_L2); }

uint64_t rs_workspace_bytes(int B, int L, int C, int H) {
  if (B < 0 || L < 1 || check_width(C) != RS_OK || check_hidden(H) != RS_OK) return 0;
  return ws_layout(static_cast<int64_t>(B) * L, C, H).total;
}

int rs_ln_stats(const void* x, int M, int C, float* stats, void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_rows(M, C, C));
  if (M == 0) return RS_OK;
  if (!x || !stats) return RS_ERR_NULL;
  if (!al16(x) || !al8(stats)) return RS_ERR_ALIGN;
  int num_sms = 148;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DevState* st = nullptr;
    RS_TRY(dev_state(&st));
    num_sms = st->num_sms;
  }
  RS_CUDA(rs::launch_ln_stats(x, M, C, stats, num_sms, static_cast<cudaStream_t>(stream)));
  return RS_OK;
}

static int ln_fc1_gelu(const void* x, int M, int C, int H, const void* W1, const void* b1,
                       const void* gamma, const void* beta, void* hidden, bool staged,
                       void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (M == 0) return RS_OK;
  if (!x || !W1 || !b1 || !gamma || !beta || !hidden) return RS_ERR_NULL;
  if (!al16(x) || !al16(W1) || !al16(b1) || !al16(gamma) || !al16(beta) || !al16(hidden))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  const WsLayout w = ws_layout(M, C, H);
  RS_TRY(ensure_ws(*st, w.fc1_total, static_cast<cudaStream_t>(stream)));
  return run_fc1(*st, x, M, C, H, W1, b1, gamma, beta, static_cast<uint8_t*>(st->ws), w, hidden,
                 staged, static_cast<cudaStream_t>(stream));
}

int rs_ln_fc1_gelu(const void* x, int M, int C, int H, const void* W1, const void* b1,
                   const void* gamma, const void* beta, void* hidden, void* stream) {
  return ln_fc1_gelu(x, M, C, H, W1, b1, gamma, beta, hidden, false, stream);
}

int rs_mlp_forward(const void* x, int M, int C, int H, const void* W1, const void* b1,
                   const void* W2, const void* b2, const void* gamma, const void* beta, void* y,
                   void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (M == 0) return RS_OK;
  if (!x || !W1 || !b1 || !W2 || !b2 || !gamma || !beta || !y) return RS_ERR_NULL;
  if (!al16(x) || !al16(W1) || !al16(b1) || !al16(W2) || !al16(b2) || !al16(gamma) ||
      !al16(beta) || !al16(y))
    return RS_ERR_ALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_mlp(*st, x, M, C, H, W1, b1, W2, b2, gamma, beta, y, s);
}

int rs_ln_fc1_gelu_staged(const void* x, int M, int C, int H, const void* W1, const void* b1,
                          const void* gamma, const void* beta, void* hidden, void* stream) {
  return ln_fc1_gelu(x, M, C, H, W1, b1, gamma, beta, hidden, true, stream);
}

int rs_ln_fold(const void* W1, const void* b1, const void* gamma, const void* beta, int C, int H,
               void* Wg, float* colG, float* colC, void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  if (!W1 || !b1 || !gamma || !beta || !Wg || !colG || !colC) return RS_ERR_NULL;
  if (!al16(W1) || !al16(gamma) || !al16(beta) || !al16(Wg) || !al4(colG) || !al4(colC))
    return RS_ERR_ALIGN;
  int num_sms = 148;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DevState* st = nullptr;
    RS_TRY(dev_state(&st));
    num_sms = st->num_sms;
  }
  RS_CUDA(rs::launch_ln_fold(W1, gamma, beta, b1, H, C, Wg, colG, colC, num_sms,
                             static_cast<cudaStream_t>(stream)));
  return RS_OK;
}

int rs_fc1_gelu_folded(const void* x, const float* stats, const void* Wg, const float* colG,
                       const float* colC, int M, int C, int H, void* hidden, void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (M == 0) return RS_OK;
  if (!x || !stats || !Wg || !colG || !colC || !hidden) return RS_ERR_NULL;
  if (!al16(x) || !al8(stats) || !al16(Wg) || !al16(colG) || !al16(colC) || !al16(hidden))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  const int bn = rs::fc1_block_n(H);
  const bool pair = rs::gemm_pair(M, C, false);
  CUtensorMap tmX, tmW, tmHid;
  RS_TRY(make_tmap(&tmX, x, C, M, 128));
  RS_TRY(make_tmap(&tmW, Wg, C, H, rs::gemm_b_box_rows(bn, pair)));
  RS_TRY(make_tmap(&tmHid, hidden, H, M, rs::kEpiBoxRows, rs::fc1_out_box_cols(H, C, false)));
  rs::MlpParams p{};
  p.M = M;
  p.N = H;
  p.K = C;
  p.n_blocks = H / bn;
  p.num_tiles = rs::gemm_num_tiles(M, p.n_blocks, pair);
  p.stats = reinterpret_cast<const float2*>(stats);
  p.colG = colG;
  p.colC = colC;
  p.out = static_cast<__nv_bfloat16*>(hidden);
  p.err = st->err;
  p.timeout_ns = rs::kDefaultTimeoutNs;
  p.debug_skip_kb = -1;
  RS_CUDA(rs::launch_fc1(tmX, tmW, tmHid, p, bn, false, pair, st->num_sms,
                         static_cast<cudaStream_t>(stream)));
  return RS_OK;
}

int rs_debug_fc1_skip_load(const void* x, int M, int C, int H, const void* W1, const void* b1,
                           const void* gamma, const void* beta, void* hidden, int skip_kblock,
                           int timeout_us, void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (M == 0) return RS_OK;
  if (skip_kblock < 0 || skip_kblock >= C / 64 || timeout_us < 1 || timeout_us > 10000000)
    return RS_ERR_SHAPE;
  if (!x || !W1 || !b1 || !gamma || !beta || !hidden) return RS_ERR_NULL;
  if (!al16(x) || !al16(W1) || !al16(b1) || !al16(gamma) || !al16(beta) || !al16(hidden))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  const WsLayout w = ws_layout(M, C, H);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  RS_TRY(ensure_ws(*st, w.fc1_total, s));
  uint8_t* ws = static_cast<uint8_t*>(st->ws);
  float* stats = reinterpret_cast<float*>(ws + w.stats);
  void* wg = ws + w.wg;
  float* colg = reinterpret_cast<float*>(ws + w.colg);
  float* colc = reinterpret_cast<float*>(ws + w.colc);
  RS_CUDA(rs::launch_ln_prep(x, M, C, stats, W1, gamma, beta, b1, H, wg, colg, colc, st->num_sms,
                             s));
  const int bn = rs::fc1_block_n(H);
  const bool pair = rs::gemm_pair(M, C, false);
  CUtensorMap tmX, tmW, tmHid;
  RS_TRY(make_tmap(&tmX, x, C, M, 128));
  RS_TRY(make_tmap(&tmW, wg, C, H, rs::gemm_b_box_rows(bn, pair)));
  RS_TRY(make_tmap(&tmHid, hidden, H, M, rs::kEpiBoxRows, rs::fc1_out_box_cols(H, C, false)));
  rs::MlpParams p{};
  p.M = M;
  p.N = H;
  p.K = C;
  p.n_blocks = H / bn;
  p.num_tiles = rs::gemm_num_tiles(M, p.n_blocks, pair);
  p.stats = reinterpret_cast<const float2*>(stats);
  p.colG = colg;
  p.colC = colc;
  p.out = static_cast<__nv_bfloat16*>(hidden);
  p.err = st->err;
  p.timeout_ns = static_cast<unsigned long long>(timeout_us) * 1000ull;
  p.debug_skip_kb = skip_kblock;
  RS_CUDA(rs::launch_fc1(tmX, tmW, tmHid, p, bn, false, pair, st->num_sms, s));
  return RS_OK;
}

int rs_mlp_fused_supported(int C, int H) { return rs::fused_supported(C, H) ? 1 : 0; }

int rs_mlp_fused(const void* x, const float* stats, const void* Wg, const float* colG,
                 const float* colC, int M, int C, int H, const void* W2, const void* b2, void* y,
                 float* partials, void* stream) {
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (!rs::fused_supported(C, H)) return RS_ERR_SHAPE;
  if (M == 0) return RS_OK;
  if (!x || !stats || !Wg || !colG || !colC || !W2 || !b2 || !y || !partials) return RS_ERR_NULL;
  if (!al16(x) || !al8(stats) || !al16(Wg) || !al16(colG) || !al16(colC) || !al16(W2) ||
      !al16(b2) || !al16(y) || !al4(partials))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_fused_step(*st, x, stats, Wg, colG, colC, M, C, H, W2, b2, y, partials,
                        static_cast<cudaStream_t>(stream), false);
}

int rs_gelu_apply(const float* z, float* out, int n, void* stream) {
  if (n < 0) return RS_ERR_SHAPE;
  if (n == 0) return RS_OK;
  if (!z || !out) return RS_ERR_NULL;
  if (!al4(z) || !al4(out)) return RS_ERR_ALIGN;
  RS_CUDA(rs::launch_gelu(z, out, n, static_cast<cudaStream_t>(stream)));
  return RS_OK;
}

int rs_fc2_residual_shift_ex(const void* hidden, const void* x, int M, int C, int H,
                             const void* W2, const void* b2, int distance, void* y,
                             float* partials, void* stream) {
  RS_TRY(check_mode(distance, 0));
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(M, C, H));
  if (M == 0) return RS_OK;
  if (!hidden || !x || !W2 || !b2 || !y || !partials) return RS_ERR_NULL;
  if (!al16(hidden) || !al16(x) || !al16(W2) || !al16(b2) || !al16(y) || !al4(partials))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_fc2(*st, hidden, x, M, C, H, W2, b2, y, partials, distance,
                 static_cast<cudaStream_t>(stream));
}
int rs_fc2_residual_shift(const void* hidden, const void* x, int M, int C, int H, const void* W2,
                          const void* b2, void* y, float* partials, void* stream) {
  return rs_fc2_residual_shift_ex(hidden, x, M, C, H, W2, b2, RS_DIST_L2, y, partials, stream);
}

int rs_select_topk_ex(const float* partials, int num_partials, int B, int L, int keep_k,
                      int distance, int flags, float* scores, int32_t* kept_idx, void* stream) {
  RS_TRY(check_mode(distance, flags));
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_partials(num_partials, distance));
  if (static_cast<int64_t>(B) * L * num_partials >= (static_cast<int64_t>(1) << 31))
    return RS_ERR_SHAPE;
  RS_TRY(check_keep(keep_k, L, flags));
  if (B == 0) return RS_OK;
  if (!partials || !scores || (!kept_idx && keep_k + !(flags & RS_NO_CLS) > 0)) return RS_ERR_NULL;
  if (!al4(partials) || !al4(scores) || !al4(kept_idx)) return RS_ERR_ALIGN;
  RS_CUDA(rs::launch_select(partials, num_partials, B, L, keep_k, distance,
                            !(flags & RS_NO_CLS), scores, kept_idx,
                            static_cast<cudaStream_t>(stream)));
  return RS_OK;
}
int rs_select_topk(const float* partials, int num_partials, int B, int L, int keep_k,
                   float* scores, int32_t* kept_idx, void* stream) {
  return rs_select_topk_ex(partials, num_partials, B, L, keep_k, RS_DIST_L2, 0, scores, kept_idx,
                           stream);
}

int rs_select_gather_ex(const float* partials, int num_partials, const void* y, int B, int L,
                        int C, int keep_k, int distance, int flags, float* scores,
                        int32_t* kept_idx, void* y_kept, void* stream) {
  RS_TRY(check_mode(distance, flags));
  RS_TRY(check_width(C));
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_partials(num_partials, distance));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, num_partials));
  RS_TRY(check_keep(keep_k, L, flags));
  if (B == 0) return RS_OK;
  if (!partials || !y || !scores ||
      (keep_k + !(flags & RS_NO_CLS) > 0 && (!kept_idx || !y_kept)))
    return RS_ERR_NULL;
  if (!al4(partials) || !al16(y) || !al4(scores) || !al4(kept_idx) || !al16(y_kept))
    return RS_ERR_ALIGN;
  int num_sms = 148;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DevState* st = nullptr;
    RS_TRY(dev_state(&st));
    num_sms = st->num_sms;
  }
  RS_CUDA(rs::launch_select_gather(partials, num_partials, y, B, L, C, keep_k, distance,
                                   !(flags & RS_NO_CLS), scores, kept_idx, y_kept, num_sms,
                                   static_cast<cudaStream_t>(stream)));
  return RS_OK;
}
int rs_select_gather(const float* partials, int num_partials, const void* y, int B, int L, int C,
                     int keep_k, float* scores, int32_t* kept_idx, void* y_kept, void* stream) {
  return rs_select_gather_ex(partials, num_partials, y, B, L, C, keep_k, RS_DIST_L2, 0, scores,
                             kept_idx, y_kept, stream);
}

int rs_gather_rows(const void* y, int B, int L, int C, const int32_t* kept_idx, int keep_k,
                   void* y_kept, void* stream) {
  RS_TRY(check_width(C));
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, C));
  if (keep_k < 0 || keep_k > L - 1) return RS_ERR_KEEP_K;
  if (B == 0) return RS_OK;
  if (!y || !kept_idx || !y_kept) return RS_ERR_NULL;
  if (!al16(y) || !al4(kept_idx) || !al16(y_kept)) return RS_ERR_ALIGN;
  int num_sms = 148;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DevState* st = nullptr;
    RS_TRY(dev_state(&st));
    num_sms = st->num_sms;
  }
  RS_CUDA(rs::launch_gather(y, B, L, C, kept_idx, keep_k + 1, y_kept, num_sms,
                            static_cast<cudaStream_t>(stream)));
  return RS_OK;
}

int rs_block_forward_ex(const void* x, int B, int L, int C, int H, const void* W1,
                        const void* b1, const void* W2, const void* b2, const void* gamma,
                        const void* beta, int keep_k, int distance, int flags, void* y_kept,
                        int32_t* kept_idx, float* scores, void* stream) {
  RS_TRY(check_mode(distance, flags));
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  const int64_t M64 = static_cast<int64_t>(B) * L;
  RS_TRY(check_rows(M64, C, H));
  RS_TRY(check_keep(keep_k, L, flags));
  if (B == 0) return RS_OK;
  const bool rows_out = keep_k + !(flags & RS_NO_CLS) > 0;  // any kept row per sample
  if (!x || !W1 || !b1 || !W2 || !b2 || !gamma || !beta || !scores ||
      (rows_out && (!y_kept || !kept_idx)))
    return RS_ERR_NULL;
  if (!al16(x) || !al16(W1) || !al16(b1) || !al16(W2) || !al16(b2) || !al16(gamma) ||
      !al16(beta) || !al16(y_kept) || !al4(kept_idx) || !al4(scores))
    return RS_ERR_ALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_block(*st, x, B, L, C, H, W1, b1, W2, b2, gamma, beta, keep_k, distance, flags,
                   y_kept, kept_idx, scores, s);
}
int rs_block_forward_block_shift_ex(const void* x_in, const void* x, int B, int L, int C, int H,
                                    const void* W1, const void* b1, const void* W2,
                                    const void* b2, const void* gamma, const void* beta,
                                    int keep_k, int distance, int flags, void* y_kept,
                                    int32_t* kept_idx, float* scores, void* stream) {
  if (B > 0 && !x_in) return RS_ERR_NULL;
  if (!al16(x_in)) return RS_ERR_ALIGN;
  RS_TRY(check_mode(distance, flags));
  if (B < 0 || L < 1 || L > RS_MAX_L) return RS_ERR_SHAPE;
  RS_TRY(check_width(C));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, H));
  RS_TRY(check_keep(keep_k, L, flags));
  if (B == 0) return RS_OK;
  const bool rows_out = keep_k + !(flags & RS_NO_CLS) > 0;
  if (!x || !W1 || !b1 || !W2 || !b2 || !gamma || !beta || !scores ||
      (rows_out && (!y_kept || !kept_idx)))
    return RS_ERR_NULL;
  if (!al16(x) || !al16(W1) || !al16(b1) || !al16(W2) || !al16(b2) || !al16(gamma) ||
      !al16(beta) || !al16(y_kept) || !al4(kept_idx) || !al4(scores))
    return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_block(*st, x, B, L, C, H, W1, b1, W2, b2, gamma, beta, keep_k, distance, flags,
                   y_kept, kept_idx, scores, static_cast<cudaStream_t>(stream), x_in);
}

int rs_block_forward(const void* x, int B, int L, int C, int H, const void* W1, const void* b1,
                     const void* W2, const void* b2, const void* gamma, const void* beta,
                     int keep_k, void* y_kept, int32_t* kept_idx, float* scores, void* stream) {
  return rs_block_forward_ex(x, B, L, C, H, W1, b1, W2, b2, gamma, beta, keep_k, RS_DIST_L2, 0,
                             y_kept, kept_idx, scores, stream);
}

int rs_attn_core(const void* qkv, int B, int L, int heads, void* out, void* stream) {
  if (B < 0 || L < 1 || L > RS_MAX_L || heads < 1) return RS_ERR_SHAPE;
  const int C = 64 * heads;
  RS_TRY(check_heads(C, heads));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, 3 * C));
  if (B == 0) return RS_OK;
  if (!qkv || !out) return RS_ERR_NULL;
  if (!al16(qkv) || !al16(out)) return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_attn_core(*st, qkv, B, L, C, heads, out, static_cast<cudaStream_t>(stream), false);
}

int rs_debug_attn_skip_load(const void* qkv, int B, int L, int heads, void* out, int skip_block,
                            int timeout_us, void* stream) {
  if (B < 0 || L < 1 || L > RS_MAX_L || heads < 1) return RS_ERR_SHAPE;
  const int C = 64 * heads;
  RS_TRY(check_heads(C, heads));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, 3 * C));
  if (skip_block < 0 || skip_block >= (L + 63) / 64 || timeout_us < 1 || timeout_us > 10000000)
    return RS_ERR_SHAPE;
  if (B == 0) return RS_OK;
  if (!qkv || !out) return RS_ERR_NULL;
  if (!al16(qkv) || !al16(out)) return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_attn_core(*st, qkv, B, L, C, heads, out, static_cast<cudaStream_t>(stream), false,
                       skip_block, static_cast<unsigned long long>(timeout_us) * 1000ull);
}

int rs_attn_sublayer(const void* x, int B, int L, int C, int heads, const void* Wqkv,
                     const void* bqkv, const void* Wo, const void* bo, const void* gamma,
                     const void* beta, void* x_out, void* stream) {
  RS_TRY(check_attn_args(x, B, L, C, heads, Wqkv, bqkv, Wo, bo, gamma, beta));
  if (B == 0) return RS_OK;
  if (!x_out) return RS_ERR_NULL;
  if (!al16(x_out)) return RS_ERR_ALIGN;
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  return run_attn_sublayer(*st, x, B, L, C, heads, Wqkv, bqkv, Wo, bo, gamma, beta, x_out,
                           RS_DIST_L2, static_cast<cudaStream_t>(stream), nullptr, nullptr);
}

int rs_attn_forward_ex(const void* x, int B, int L, int C, int heads, const void* Wqkv,
                       const void* bqkv, const void* Wo, const void* bo, const void* gamma,
                       const void* beta, int keep_k, int distance, int flags, void* x_kept,
                       int32_t* kept_idx, float* scores, void* stream) {
  RS_TRY(check_mode(distance, flags));
  RS_TRY(check_attn_args(x, B, L, C, heads, Wqkv, bqkv, Wo, bo, gamma, beta));
  RS_TRY(check_keep(keep_k, L, flags));
  if (B == 0) return RS_OK;
  const bool rows_out = keep_k + !(flags & RS_NO_CLS) > 0;
  if (!scores || (rows_out && (!x_kept || !kept_idx))) return RS_ERR_NULL;
  if (!al16(x_kept) || !al4(kept_idx) || !al4(scores)) return RS_ERR_ALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  uint8_t* ws = nullptr;
  WsLayout w{};
  RS_TRY(run_attn_sublayer(*st, x, B, L, C, heads, Wqkv, bqkv, Wo, bo, gamma, beta, nullptr,
                           distance, s, &ws, &w));
  const int np =
      rs::dist_partials(distance) * rs::kFc2PartialsPerTile * C / rs::fc2_block_n(C);
  RS_CUDA(rs::launch_select_gather(reinterpret_cast<float*>(ws + w.partials), np, ws + w.y, B, L,
                                   C, keep_k, distance, !(flags & RS_NO_CLS), scores, kept_idx,
                                   x_kept, st->num_sms, s, /*pdl=*/true));
  return RS_OK;
}

int rs_encoder_forward(const void* x, int B, int L, int C, int H, int heads, int depth,
                       const void* const* weights, const int* keep, void* out, void* stream) {
  if (B < 0 || L < 1 || L > RS_MAX_L || depth < 1 || depth > 1024) return RS_ERR_SHAPE;
  RS_TRY(check_heads(C, heads));
  RS_TRY(check_hidden(H));
  RS_TRY(check_rows(static_cast<int64_t>(B) * L, C, H > 3 * C ? H : 3 * C));
  if (!weights || !keep) return RS_ERR_NULL;
  int Lc = L;
  for (int l = 0; l < depth; ++l) {
    if (keep[l] >= 0) {
      RS_TRY(check_keep(keep[l], Lc, 0));
      Lc = 1 + keep[l];
    }
  }
  if (B == 0) return RS_OK;
  if (!x || !out) return RS_ERR_NULL;
  if (!al16(x) || !al16(out)) return RS_ERR_ALIGN;
  for (int i = 0; i < 12 * depth; ++i) {
    if (!weights[i]) return RS_ERR_NULL;
    if (!al16(weights[i])) return RS_ERR_ALIGN;
  }
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  // activations: x' and two ping-pong layer outputs [B, L, C] bf16, then the
  // kept indices and scores of a pruning layer
  const size_t xb = align_up(static_cast<size_t>(B) * L * C * 2, 1024);
  const size_t ib = align_up(static_cast<size_t>(B) * L * 4, 1024);
  RS_TRY(ensure_act(*st, 3 * xb + 2 * ib, s));
  uint8_t* act = static_cast<uint8_t*>(st->act);
  void* xp = act;
  void* buf[2] = {act + xb, act + 2 * xb};
  int32_t* kept = reinterpret_cast<int32_t*>(act + 3 * xb);
  float* scores = reinterpret_cast<float*>(act + 3 * xb + ib);
  // the largest workspace any layer needs, once, before the first launch
  {
    const int64_t M = static_cast<int64_t>(B) * L;
    const size_t a = attn_ws_layout(M, C).w.total, m = ws_layout(M, C, H).total;
    RS_TRY(ensure_ws(*st, a > m ? a : m, s));
  }
  const void* cur = x;
  Lc = L;
  for (int l = 0; l < depth; ++l) {
    const void* const* w = weights + 12 * l;
    void* nxt = l + 1 == depth ? out : buf[l & 1];
    RS_TRY(run_attn_sublayer(*st, cur, B, Lc, C, heads, w[0], w[1], w[2], w[3], w[4], w[5], xp,
                             RS_DIST_L2, s, nullptr, nullptr));
    if (keep[l] >= 0) {
      RS_TRY(run_block(*st, xp, B, Lc, C, H, w[6], w[7], w[8], w[9], w[10], w[11], keep[l],
                       RS_DIST_L2, 0, nxt, kept, scores, s));
      Lc = 1 + keep[l];
    } else {
      RS_TRY(run_mlp(*st, xp, B * Lc, C, H, w[6], w[7], w[8], w[9], w[10], w[11], nxt, s));
    }
    cur = nxt;
  }
  return RS_OK;
}

int rs_get_last_device_error(void* stream) {
  std::lock_guard<std::mutex> lock(g_mu);
  DevState* st = nullptr;
  RS_TRY(dev_state(&st));
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  int v = 0;
  RS_CUDA(cudaMemcpy(&v, st->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) RS_CUDA(cudaMemset(st->err, 0, sizeof(int)));
  // rs_ln_fc1_gelu_noalloc records its status in its own static scratch
  const int na = rs::noalloc_take_error();
  return v != 0 ? v : na;
}

void rs_release_workspace(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return;
  for (int d = 0; d < kMaxDevices; ++d) {
    DevState& st = g_dev[d];
    if (st.ws == nullptr && st.act == nullptr) continue;
    if (cudaSetDevice(d) == cudaSuccess) {
      cudaDeviceSynchronize();
      if (st.ws) cudaFreeAsync(st.ws, 0);
      if (st.act) cudaFreeAsync(st.act, 0);
      cudaDeviceSynchronize();
      cudaGetLastError();
    }
    st.ws = nullptr;
    st.ws_bytes = 0;
    st.act = nullptr;
    st.act_bytes = 0;
  }
  cudaSetDevice(cur);
}

}  // extern "C"
