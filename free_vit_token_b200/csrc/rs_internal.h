// rs_internal.h -- declarations shared by the library's translation units
// (kernel parameter blocks and host-side launchers). Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rs.h"

namespace rs {

constexpr float kLnEps = 1e-6f;          // LayerNorm epsilon (the pages do not state one)
constexpr int kEpiGelu = 0;              // fc1 epilogue: + b1, erf-GELU, bf16 store
constexpr int kEpiResidShift = 1;        // fc2 epilogue: + b2, residual, shift partials
constexpr int kEpiGeluFold = 2;          // fc1 epilogue: folded LN (mean, rstd, G, cb), erf-GELU
constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;  // one pipeline wait: 4 s
// The GEMM epilogue reads its accumulators 16 columns at a time and writes its
// outputs (hidden, y) through per-warp boxes of 32 rows and up to kEpiBoxMaxCols
// bf16 columns (a 64-byte swizzled row), one TMA store per box: wider boxes move
// the output in fewer row transfers, which the operand loads share the TMA unit
// with. Output tensor maps use the box of out_box_cols.
constexpr int kEpiBoxRows = 32;
constexpr int kEpiChunkCols = 16;
constexpr int kEpiBoxMaxCols = 32;
// Epilogue warps of the GEMM kernels: 16 for the folded-LN fc1 with a short
// reduction (K <= 512), whose epilogue rivals the main loop; 8 otherwise.
__host__ __device__ constexpr int gemm_epi_warps(bool folded_fc1, int K) {
  return folded_fc1 && K <= 512 ? 16 : 8;
}
// Output box width for tiles of bn columns and ew epilogue warps (each warp owns
// bn / (ew / 4) columns of a tile).
__host__ __device__ constexpr int out_box_cols(int bn, int ew) {
  return bn * 4 / ew < kEpiBoxMaxCols ? bn * 4 / ew : kEpiBoxMaxCols;
}
// fc2 writes this many shift partials per row and 128 x BN output tile (one per
// epilogue column group).
constexpr int kFc2PartialsPerTile = 2;
// Shift distances (§3.3 "Distance metrics"): the values of rs.h's RS_DIST_*. fc2
// writes one partial per column group for L2 (sum of squares) and L1 (sum of
// absolute values), three for cosine (sum h.x, sum h.h, sum x.x).
constexpr int kDistL2 = 0;
constexpr int kDistL1 = 1;
constexpr int kDistCos = 2;
inline int dist_partials(int dist) { return dist == kDistCos ? 3 : 1; }

// Launches `kern` on `stream`; with `pdl` the launch may begin while the
// previous kernel in the stream is still running (every kernel of this library
// waits for its predecessor with griddepcontrol.wait before touching memory).
// With `cluster` > 1 the grid is cut into clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, bool pdl, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = n > 0 ? attr : nullptr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool pdl, Args&&... args) {
  return launch_cluster(kern, grid, block, smem, stream, pdl, 1, static_cast<Args&&>(args)...);
}

struct MlpParams {
  int M, N, K;                    // output rows, output columns, reduction length
  int n_blocks, num_tiles;        // N / BN, gemm_num_tiles(M, n_blocks, pair)
  const __nv_bfloat16* ln_gamma;  // [K]   fc1 only
  const __nv_bfloat16* ln_beta;   // [K]   fc1 only
  const float2* stats;            // [M]   fc1 only: (mean, rstd) per row
  const float* colG;              // [N]   folded-LN fc1: sum_c Wg[j, c]
  const float* colC;              // [N]   folded-LN fc1: sum_c W1[j, c] beta[c] + b1[j]
  const __nv_bfloat16* bias;      // [N]
  __nv_bfloat16* out;             // [M, N] hidden (fc1) or y (fc2)
  const __nv_bfloat16* resid;     // [M, N] x' (fc2 only)
  float* partials;                // [M, num_partials] (fc2 only)
  int num_partials;               // 2 * n_blocks (fc2)
  int* err;                       // device status flag
  unsigned long long timeout_ns;  // limit of one pipeline wait
  int debug_skip_kb;              // test hook: CTA 0 skips this k-block's loads of its
                                  // first tile (-1: off)
  int dist;                       // fc2: kDistL2, kDistL1 or kDistCos
  int linear;                     // folded-LN fc1: 0 = erf-GELU, 1 = no activation (QKV)
  const __nv_bfloat16* shift_ref; // fc2: null, or [M, N]: the shift compares y = x' + h with
                                  // this block input instead of h with x' (§3.3 case (iii))
};

size_t mlp_smem_bytes(int bn, bool ln, int epi, int K, int ew, bool pair = false);

// The driver's cuTensorMapEncodeTiled (resolved once through the runtime), or null.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
// Row-major bf16 [rows, inner] viewed as tiles of {box_inner elements, box_rows
// rows}: 64-wide boxes use the 128-byte swizzle (GEMM operands), 16-wide boxes
// the 32-byte swizzle (epilogue output boxes). Rows past the end read as zero
// and are not written. Returns RS_OK or RS_ERR_CUDA.
int make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows,
              uint32_t box_inner = 64);
// rs_ln_fc1_gelu_noalloc's status slot on the current device: returns it (RS_OK or
// RS_ERR_DEVICE_TIMEOUT) and clears it, RS_OK when that entry point never ran on
// this device, RS_ERR_CUDA when the read fails. The caller has synchronised.
int noalloc_take_error();

// CTA pairs (tcgen05 cta_group::2, 256-row tiles with B split between the two
// CTAs) for long reductions (K >= 1024: fc2, and fc1 at C >= 1024), where the
// third less operand traffic per CTA pays; single CTAs (128-row tiles) for short
// K, where the epilogue bounds the kernel and one tile per SM (148 units rather
// than the resident pairs) splits the grid into fewer waves. Not for the
// staged-LN kernel.
inline bool gemm_pair(int M, int K, bool staged_ln) { return !staged_ln && M > 128 && K >= 1024; }
inline int gemm_num_tiles(int M, int n_blocks, bool pair) {
  const int tm = pair ? 256 : 128;
  return ((M + tm - 1) / tm) * n_blocks;
}
// Rows of the B tile one CTA loads (its tensor map's box height).
inline int gemm_b_box_rows(int bn, bool pair) { return pair ? bn / 2 : bn; }
int fc1_block_n(int H);
int fc2_block_n(int C);
// Output box columns of the fc1 kernel for these sizes (staged: the staged-LN
// kernel) and of the fc2 kernel.
inline int fc1_out_box_cols(int H, int C, bool staged) {
  return out_box_cols(fc1_block_n(H), staged ? 8 : gemm_epi_warps(true, C));
}
inline int fc2_out_box_cols(int C) { return out_box_cols(fc2_block_n(C), 8); }
cudaError_t launch_ln_stats(const void* x, int M, int C, float* stats, int num_sms,
                            cudaStream_t stream, bool pdl = false);
cudaError_t launch_ln_fold(const void* W1, const void* gamma, const void* beta, const void* b1,
                           int H, int C, void* Wg, float* colG, float* colC, int num_sms,
                           cudaStream_t stream, bool pdl = false);
// LN statistics of x' and the fold of gamma, beta into W1, in one launch.
cudaError_t launch_ln_prep(const void* x, int M, int C, float* stats, const void* W1,
                           const void* gamma, const void* beta, const void* b1, int H, void* Wg,
                           float* colG, float* colC, int num_sms, cudaStream_t stream,
                           bool pdl = false);
// `pair`: CTA-pair kernel (p.num_tiles and tmW1's box from gemm_num_tiles and
// gemm_b_box_rows with the same flag); not with staged_ln.
cudaError_t launch_fc1(const CUtensorMap& tmX, const CUtensorMap& tmW1, const CUtensorMap& tmHid,
                       const MlpParams& p, int bn, bool staged_ln, bool pair, int num_sms,
                       cudaStream_t s, bool pdl = false);
cudaError_t launch_gelu(const float* z, float* out, int n, cudaStream_t stream);
cudaError_t launch_fc2(const CUtensorMap& tmHid, const CUtensorMap& tmW2, const CUtensorMap& tmY,
                       const MlpParams& p, int bn, bool pair, int num_sms, cudaStream_t s,
                       bool pdl = false);
// The fused MLP kernel (rs_fused.cu): fc1, GELU, fc2, residual and shift partials
// in one kernel, for narrow blocks.
constexpr int kFusedMaxC = 384;    // fc2's fp32 accumulator (C columns) + 128 in TMEM
constexpr int kFusedPartials = 4;  // shift partials per row (one per column quarter)
inline bool fused_supported(int C, int H) {
  return C >= 64 && C % 64 == 0 && C <= kFusedMaxC && H >= 128 && H % 128 == 0;
}
struct FusedParams {
  int M, C, H, num_m;             // rows, width, hidden width, ceil(M / 128)
  const float2* stats;            // [M] (mean, rstd)
  const float* colG;              // [H] sum_c Wg[j, c]
  const float* colC;              // [H] sum_c W1[j, c] beta[c] + b1[j]
  const __nv_bfloat16* b2;        // [C]
  const __nv_bfloat16* x;         // [M, C] x' (residual)
  float* partials;                // [M, kFusedPartials]
  int* err;                       // device status flag
  unsigned long long timeout_ns;  // limit of one pipeline wait
};
// Rows of W2 per TMA box and fc2 MMA (N): 128 when C is a multiple of 128, else 64.
int fused_w2_rows(int C);
// tmX: x' [M, C], box 64 x 128; tmWg: Wg [H, C], box 64 x 128; tmW2: W2 [C, H], box
// 64 x fused_w2_rows(C); tmY: y [M, C], box 16 x 32 (the 32-byte swizzle).
cudaError_t launch_mlp_fused(const CUtensorMap& tmX, const CUtensorMap& tmWg,
                             const CUtensorMap& tmW2, const CUtensorMap& tmY, const FusedParams& p,
                             int num_sms, cudaStream_t stream, bool pdl = false);

// Selection: `dist` says how partials make a score (kDist*), `cls` whether t = 0 is a
// CLS token (kept first, never ranked) or ranked like the others. kept_idx holds
// cls + keep_k entries per sample.
cudaError_t launch_select(const float* partials, int num_partials, int B, int L, int keep_k,
                          int dist, bool cls, float* scores, int32_t* kept_idx,
                          cudaStream_t stream, bool pdl = false);
// Gathers k1 rows per sample (k1 = entries of kept_idx per sample).
cudaError_t launch_gather(const void* y, int B, int L, int C, const int32_t* kept_idx, int k1,
                          void* y_kept, int num_sms, cudaStream_t stream, bool pdl = false);
// Selection then gather in one kernel (B x S CTAs; every CTA of a sample selects).
cudaError_t launch_select_gather(const float* partials, int num_partials, const void* y, int B,
                                 int L, int C, int keep_k, int dist, bool cls, float* scores,
                                 int32_t* kept_idx, void* y_kept, int num_sms,
                                 cudaStream_t stream, bool pdl = false);

// Attention core (rs_attn.cu): per sample and head of width 64, Softmax(Q K^T / 8) V
// from a QKV projection [B, L, 3C] (Q, K, V at columns 0, C, 2C; head h at +64 h),
// written to out [B, L, C] (head h at columns 64 h). Both tensor maps view the
// QKV buffer as [B][L][3C] with the 128-byte swizzle, in boxes of {64,
// attn_q_box_rows(), 1} (Q) and {64, attn_kv_box_rows(), 1} (K and V).
struct AttnParams {
  int B, L, C, heads;
  __nv_bfloat16* out;
  int* err;                       // device status flag
  unsigned long long timeout_ns;  // limit of one pipeline wait
  int debug_skip_block;           // test hook: CTA (0, 0, 0) withholds this key block's
                                  // loads and every later one (-1: off)
};
size_t attn_smem_bytes();
int attn_q_box_rows();
int attn_kv_box_rows();
cudaError_t launch_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKV, const AttnParams& p,
                        cudaStream_t stream, bool pdl = false);

}  // namespace rs
