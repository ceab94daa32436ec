// rs_ln.cu -- the LayerNorm pieces of the MLP sublayer (§3.3 Eq. (6) of
// "Representation Shift: Unifying Token Compression with FlashAttention"):
//
//   ln_stats:  per row r of x', mean_r and rstd_r = 1/sqrt(var_r + eps) (biased
//              variance), 8, 16 or 32 lanes per row by width, two passes over
//              the row held in registers, reductions by shuffles.
//   ln_fold:   the LayerNorm's affine part folded into fc1's weights. With
//              u = (x' - mean) * rstd * gamma + beta,
//                W1 u + b1 = rstd * (Wg x' - mean * G) + cb,
//              Wg[j, c] = bf16(W1[j, c] * gamma[c]), G[j] = sum_c Wg[j, c],
//              cb[j] = sum_c W1[j, c] * beta[c] + b1[j]. G is summed from the
//              rounded Wg so that the mean cancels exactly in exact arithmetic.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rs_internal.h"
#include "rs_ptx.cuh"

namespace rs {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Persistent: each warp takes 32 / LPR rows per step (LPR lanes per row, VPL
// 16-byte vectors per lane at most), walks the rows with a grid-wide stride and
// keeps the next step's loads in flight while it reduces the current rows. Sums
// run on pairs of fp32 lanes. `gw0`/`nw` are this warp's index and the warp
// count of the part of the grid doing this work.
template <int LPR, int VPL>
__device__ __forceinline__ void ln_stats_body(const __nv_bfloat16* __restrict__ x, int M, int C,
                                              float2* __restrict__ stats, int gw0, int nw) {
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, l = lane % LPR;
  const int nvec = C >> 3;
  const float inv_c = 1.0f / static_cast<float>(C);
  auto load = [&](int r, uint4(&v)[VPL]) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * C);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = l + LPR * i;
      v[i] = (r < M && idx < nvec) ? __ldg(xr + idx) : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 cur[VPL], nxt[VPL];
  const int step = nw * RPW;
  int base = gw0 * RPW;
  if (base < M) load(base + sub, cur);
  for (; base < M; base += step) {
    const int row = base + sub;
    if (base + step < M) load(base + step + sub, nxt);
    uint64_t s2 = 0;  // padding vectors are zero: they add nothing
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&cur[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) s2 = fadd2(s2, bf16x2_to_f2(w[e]));
    }
    float2 sf = f2unpack(s2);
    float sum = sf.x + sf.y;
#pragma unroll
    for (int o = LPR / 2; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mean = sum * inv_c;
    const uint64_t nm2 = f2pack(-mean, -mean);
    uint64_t q2 = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (l + LPR * i < nvec) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&cur[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t d2 = fadd2(bf16x2_to_f2(w[e]), nm2);
          q2 = ffma2(d2, d2, q2);
        }
      }
    }
    const float2 qf = f2unpack(q2);
    float sq = qf.x + qf.y;
#pragma unroll
    for (int o = LPR / 2; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (l == 0 && row < M) stats[row] = make_float2(mean, rsqrtf(sq * inv_c + kLnEps));
#pragma unroll
    for (int i = 0; i < VPL; ++i) cur[i] = nxt[i];
  }
}

template <int LPR, int VPL>
__global__ void __launch_bounds__(256) ln_stats_kernel(const __nv_bfloat16* __restrict__ x, int M,
                                                       int C, float2* __restrict__ stats) {
  pdl_trigger();
  pdl_wait();
  ln_stats_body<LPR, VPL>(x, M, C, stats,
                          static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5),
                          static_cast<int>((gridDim.x * blockDim.x) >> 5));
}

template <int VPL>
__device__ __forceinline__ void ln_fold_body(const __nv_bfloat16* __restrict__ W1,
                                             const __nv_bfloat16* __restrict__ gamma,
                                             const __nv_bfloat16* __restrict__ beta,
                                             const __nv_bfloat16* __restrict__ b1, int H, int C,
                                             __nv_bfloat16* __restrict__ Wg, float* __restrict__ colG,
                                             float* __restrict__ colC, int gw0, int nw) {
  const int lane = threadIdx.x & 31;
  const int nvec = C >> 3;
  const uint4* g4 = reinterpret_cast<const uint4*>(gamma);
  const uint4* b4 = reinterpret_cast<const uint4*>(beta);
  for (int j = gw0; j < H; j += nw) {
    const uint4* wr = reinterpret_cast<const uint4*>(W1 + static_cast<size_t>(j) * C);
    uint4* out = reinterpret_cast<uint4*>(Wg + static_cast<size_t>(j) * C);
    // the row's weights first (HBM), then gamma and beta (L1/L2-resident, re-read per
    // row rather than held in registers, so that the kernel keeps its occupancy)
    uint4 wv[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = lane + 32 * i;
      wv[i] = idx < nvec ? __ldg(wr + idx) : make_uint4(0, 0, 0, 0);
    }
    float gs = 0.f, cs = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = lane + 32 * i;
      if (idx < nvec) {
        const uint4 gq = __ldg(g4 + idx), bq = __ldg(b4 + idx);
        const uint32_t* w = reinterpret_cast<const uint32_t*>(&wv[i]);
        const uint32_t* g = reinterpret_cast<const uint32_t*>(&gq);
        const uint32_t* b = reinterpret_cast<const uint32_t*>(&bq);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float w0 = bf16lo(w[e]), w1 = bf16hi(w[e]);
          o[e] = pack_bf16x2(w0 * bf16lo(g[e]), w1 * bf16hi(g[e]));
          gs += bf16lo(o[e]) + bf16hi(o[e]);
          cs = fmaf(w0, bf16lo(b[e]), cs);
          cs = fmaf(w1, bf16hi(b[e]), cs);
        }
        out[idx] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
    gs = warp_sum(gs);
    cs = warp_sum(cs);
    if (lane == 0) {
      colG[j] = gs;
      colC[j] = cs + __bfloat162float(b1[j]);
    }
  }
}

template <int VPL>
__global__ void __launch_bounds__(256)
    ln_fold_kernel(const __nv_bfloat16* __restrict__ W1, const __nv_bfloat16* __restrict__ gamma,
                   const __nv_bfloat16* __restrict__ beta, const __nv_bfloat16* __restrict__ b1,
                   int H, int C, __nv_bfloat16* __restrict__ Wg, float* __restrict__ colG,
                   float* __restrict__ colC) {
  pdl_trigger();
  pdl_wait();
  ln_fold_body<VPL>(W1, gamma, beta, b1, H, C, Wg, colG, colC,
                    static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5),
                    static_cast<int>((gridDim.x * blockDim.x) >> 5));
}

// Both in one grid: the first `stats_blocks` blocks compute statistics, the rest fold.
template <int VPL, int LPR, int SVPL>
__global__ void __launch_bounds__(256)
    ln_prep_kernel(const __nv_bfloat16* __restrict__ x, int M, float2* __restrict__ stats,
                   int stats_blocks, const __nv_bfloat16* __restrict__ W1,
                   const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                   const __nv_bfloat16* __restrict__ b1, int H, int C,
                   __nv_bfloat16* __restrict__ Wg, float* __restrict__ colG,
                   float* __restrict__ colC) {
  pdl_trigger();
  pdl_wait();
  const int wpb = blockDim.x >> 5;
  const int w = threadIdx.x >> 5;
  if (static_cast<int>(blockIdx.x) < stats_blocks) {
    ln_stats_body<LPR, SVPL>(x, M, C, stats, blockIdx.x * wpb + w, stats_blocks * wpb);
  } else {
    const int fb = blockIdx.x - stats_blocks;
    ln_fold_body<VPL>(W1, gamma, beta, b1, H, C, Wg, colG, colC, fb * wpb + w,
                      (gridDim.x - stats_blocks) * wpb);
  }
}

static int stats_blocks_for(int M, int C, int num_sms) {
  const int rpw = C <= 256 ? 4 : (C <= 512 ? 2 : 1);  // rows per warp step
  const int warps = (M + 2 * rpw - 1) / (2 * rpw);    // about two steps per warp
  int blocks = (warps + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  return blocks < 1 ? 1 : blocks;
}
static int fold_blocks_for(int H, int num_sms) {
  int blocks = (H + 7) / 8;
  if (blocks > num_sms * 4) blocks = num_sms * 4;
  return blocks < 1 ? 1 : blocks;
}

cudaError_t launch_ln_stats(const void* x, int M, int C, float* stats, int num_sms,
                            cudaStream_t stream, bool pdl) {
  const int blocks = stats_blocks_for(M, C, num_sms);
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* sp = reinterpret_cast<float2*>(stats);
  if (C <= 256) return launch(ln_stats_kernel<8, 4>, blocks, 256, 0, stream, pdl, xp, M, C, sp);
  if (C <= 512) return launch(ln_stats_kernel<16, 4>, blocks, 256, 0, stream, pdl, xp, M, C, sp);
  if (C <= 1024) return launch(ln_stats_kernel<32, 4>, blocks, 256, 0, stream, pdl, xp, M, C, sp);
  return launch(ln_stats_kernel<32, 8>, blocks, 256, 0, stream, pdl, xp, M, C, sp);
}

cudaError_t launch_ln_fold(const void* W1, const void* gamma, const void* beta, const void* b1,
                           int H, int C, void* Wg, float* colG, float* colC, int num_sms,
                           cudaStream_t stream, bool pdl) {
  const int blocks = fold_blocks_for(H, num_sms);
  const auto* w = static_cast<const __nv_bfloat16*>(W1);
  const auto* g = static_cast<const __nv_bfloat16*>(gamma);
  const auto* b = static_cast<const __nv_bfloat16*>(beta);
  const auto* bb = static_cast<const __nv_bfloat16*>(b1);
  auto* o = static_cast<__nv_bfloat16*>(Wg);
  if (C <= 256)
    return launch(ln_fold_kernel<1>, blocks, 256, 0, stream, pdl, w, g, b, bb, H, C, o, colG, colC);
  if (C <= 512)
    return launch(ln_fold_kernel<2>, blocks, 256, 0, stream, pdl, w, g, b, bb, H, C, o, colG, colC);
  if (C <= 1024)
    return launch(ln_fold_kernel<4>, blocks, 256, 0, stream, pdl, w, g, b, bb, H, C, o, colG, colC);
  return launch(ln_fold_kernel<8>, blocks, 256, 0, stream, pdl, w, g, b, bb, H, C, o, colG, colC);
}

cudaError_t launch_ln_prep(const void* x, int M, int C, float* stats, const void* W1,
                           const void* gamma, const void* beta, const void* b1, int H, void* Wg,
                           float* colG, float* colC, int num_sms, cudaStream_t stream, bool pdl) {
  const int sb = stats_blocks_for(M, C, num_sms);
  const int fb = fold_blocks_for(H, num_sms);
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* sp = reinterpret_cast<float2*>(stats);
  const auto* w = static_cast<const __nv_bfloat16*>(W1);
  const auto* g = static_cast<const __nv_bfloat16*>(gamma);
  const auto* b = static_cast<const __nv_bfloat16*>(beta);
  const auto* bb = static_cast<const __nv_bfloat16*>(b1);
  auto* o = static_cast<__nv_bfloat16*>(Wg);
  const dim3 grid(sb + fb);
  if (C <= 256)
    return launch(ln_prep_kernel<1, 8, 4>, grid, 256, 0, stream, pdl, xp, M, sp, sb, w, g, b, bb, H, C, o,
                  colG, colC);
  if (C <= 512)
    return launch(ln_prep_kernel<2, 16, 4>, grid, 256, 0, stream, pdl, xp, M, sp, sb, w, g, b, bb, H, C, o,
                  colG, colC);
  if (C <= 1024)
    return launch(ln_prep_kernel<4, 32, 4>, grid, 256, 0, stream, pdl, xp, M, sp, sb, w, g, b, bb, H, C, o,
                  colG, colC);
  return launch(ln_prep_kernel<8, 32, 8>, grid, 256, 0, stream, pdl, xp, M, sp, sb, w, g, b, bb, H, C, o,
                colG, colC);
}

}  // namespace rs
