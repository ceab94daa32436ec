// rs_mlp.cu -- the two contractions of the MLP sublayer (§3.3 Eq. (6) of
// "Representation Shift: Unifying Token Compression with FlashAttention") as
// persistent, warp-specialised tcgen05 GEMMs for sm_100a, plus the LayerNorm
// row-statistics pass that feeds fc1's operand staging.
//
//   fc1:  a = GELU(LN(x') W1^T + b1)           A = x' tiles (TMA), normalised
//                                              in shared memory by LN warps
//   fc2:  h = a W2^T + b2; y = x' + h;          A = a tiles (TMA)
//         P[r, j] = sum_{c in group j} (h - x')^2   -- Eq. (4) with D = L2
//
// One CTA per SM loops over 128 x BN output tiles. Warp roles:
//   warp 0      TMA producer (A and B tiles, 64-wide K blocks, STAGES deep ring)
//   warp 1      TMEM owner and UMMA issuer (tcgen05.mma, M=128, N=BN, K=16)
//   warps 4-11  epilogue: TMEM -> registers -> bias/GELU or residual/shift -> HBM
//   warps 12-15 (fc1 only) LayerNorm staging of the A tile in place
// The fp32 accumulator is double-buffered in TMEM (2 x BN columns) so the
// epilogue of one tile overlaps the main loop of the next.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rs_internal.h"
#include "rs_ptx.cuh"

namespace rs {

constexpr int kBM = 128;
constexpr int kBK = 64;                         // one 128-byte swizzle row of bf16
constexpr int kAStageBytes = kBM * kBK * 2;     // 16 KB
constexpr int kEpiWarp0 = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kLnWarp0 = 12;
constexpr int kNumLnWarps = 4;
constexpr int kSmemLimit = 232448;              // 227 KB opt-in per CTA
constexpr int kCtrlBytes = 512;                 // barriers, TMEM slot, abort flag
constexpr uint32_t kTmemCols = 512;

__host__ __device__ constexpr int stage_bytes(int bn) { return kAStageBytes + bn * kBK * 2; }
__host__ __device__ constexpr int num_stages(int bn, bool ln) {
  // LN mode keeps gamma and beta (RS_MAX_C floats each) in shared memory too.
  return ((kSmemLimit - 1024 - kCtrlBytes - (ln ? 2 * RS_MAX_C * 4 : 0)) / stage_bytes(bn)) > 6
             ? 6
             : ((kSmemLimit - 1024 - kCtrlBytes - (ln ? 2 * RS_MAX_C * 4 : 0)) / stage_bytes(bn));
}
__host__ __device__ constexpr int num_threads(bool ln) { return (ln ? 16 : 12) * 32; }

size_t mlp_smem_bytes(int bn, bool ln, int K) {
  return 1024 + static_cast<size_t>(num_stages(bn, ln)) * stage_bytes(bn) + kCtrlBytes +
         (ln ? 2 * static_cast<size_t>(K) * 4 : 0);
}

__device__ __forceinline__ float gelu_erf(float z) {
  // exact GELU: z * Phi(z) = z/2 * (1 + erf(z / sqrt 2))
  const float hz = 0.5f * z;
  return fmaf(hz, erff(z * 0.70710678118654752f), hz);
}

template <int BN, bool LN_A, int EPI>
__global__ void __launch_bounds__(num_threads(LN_A), 1)
    mlp_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const MlpParams p) {
  constexpr int kBStageBytes = BN * kBK * 2;
  constexpr int STAGES = num_stages(BN, LN_A);
  constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, BN);
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(2 * BN <= static_cast<int>(kTmemCols), "TMEM double buffer");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kAStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * kBStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* aready = empty + STAGES;
  uint64_t* tfull = aready + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_gamma = reinterpret_cast<float*>(sB + STAGES * kBStageBytes + kCtrlBytes);
  float* s_beta = s_gamma + p.K;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&aready[s], kNumLnWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kNumEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if constexpr (LN_A) {
    for (int i = threadIdx.x; i < p.K; i += blockDim.x) {
      s_gamma[i] = __bfloat162float(p.ln_gamma[i]);
      s_beta[i] = __bfloat162float(p.ln_beta[i]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pend[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) pend[s] = -1;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        const int m_blk = tile / p.n_blocks, n_blk = tile % p.n_blocks;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], stage_bytes(BN));
          tma_load_2d(sA + stage * kAStageBytes, &tmA, &full[stage], kb * kBK, m_blk * kBM);
          tma_load_2d(sB + stage * kBStageBytes, &tmB, &full[stage], kb * kBK, n_blk * BN);
#pragma unroll
          for (int s = 0; s < STAGES; ++s)
            if (s == stage) pend[s] = static_cast<int>(phase);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // Every load this thread issued must land before the CTA may exit.
#pragma unroll
      for (int s = 0; s < STAGES; ++s)
        if (pend[s] >= 0) wait_bounded(&full[s], static_cast<uint32_t>(pend[s]), wc, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, wc)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_bounded(&full[stage], phase, wc)) { ok = false; break; }
          if (LN_A && !wait_bounded(&aready[stage], phase, wc)) { ok = false; break; }
          tc_fence_after_sync();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * kAStageBytes));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * kBStageBytes));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, ad + 2u * k, bd + 2u * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
          issued = true;
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (*abort_flag && issued) {
        // Drain: wait until every MMA issued so far has finished with TMEM and smem.
        umma_commit(drain);
        wait_bounded(drain, 0u, wc, false);
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                          // TMEM lane quadrant of this warp
    const int half = (warp - kEpiWarp0) >> 2;        // which half of the BN columns
    constexpr int kHalf = BN / 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int m_blk = tile / p.n_blocks, n_blk = tile % p.n_blocks;
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, wc) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      mbar_try_wait(&tfull[acc], acc_phase);  // completed: acquire for every lane
      tc_fence_after_sync();
      const int row = m_blk * kBM + q * 32 + lane;
      const bool row_ok = row < p.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * kHalf);
      const int col0 = n_blk * BN + half * kHalf;
      float part = 0.f;
#pragma unroll 1
      for (int c = 0; c < kHalf; c += 32) {
        uint32_t r[32];
        tmem_load_32cols(t_row + c, r);
        const uint4* bptr = reinterpret_cast<const uint4*>(p.bias + col0 + c);
        uint4 bv[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) bv[v] = __ldg(bptr + v);
        const uint32_t* bw = reinterpret_cast<const uint32_t*>(bv);
        uint32_t outw[16];
        if constexpr (EPI == kEpiGelu) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float z0 = __uint_as_float(r[2 * e]) + bf16lo(bw[e]);
            const float z1 = __uint_as_float(r[2 * e + 1]) + bf16hi(bw[e]);
            outw[e] = pack_bf16x2(gelu_erf(z0), gelu_erf(z1));
          }
        } else {
          uint4 xv[4] = {};
          const size_t off = static_cast<size_t>(row) * p.N + col0 + c;
          if (row_ok) {
            const uint4* xptr = reinterpret_cast<const uint4*>(p.resid + off);
#pragma unroll
            for (int v = 0; v < 4; ++v) xv[v] = __ldg(xptr + v);
          }
          const uint32_t* xw = reinterpret_cast<const uint32_t*>(xv);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float x0 = bf16lo(xw[e]), x1 = bf16hi(xw[e]);
            const float h0 = __uint_as_float(r[2 * e]) + bf16lo(bw[e]);
            const float h1 = __uint_as_float(r[2 * e + 1]) + bf16hi(bw[e]);
            outw[e] = pack_bf16x2(x0 + h0, x1 + h1);
            const float d0 = h0 - x0, d1 = h1 - x1;
            part = fmaf(d0, d0, part);
            part = fmaf(d1, d1, part);
          }
        }
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(row) * p.N + col0 + c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
        }
      }
      if constexpr (EPI == kEpiResidShift) {
        if (row_ok) p.partials[static_cast<size_t>(row) * p.num_partials + n_blk * 2 + half] = part;
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  } else if (LN_A && warp >= kLnWarp0) {
    // ------------------------------------------------------------ LayerNorm staging
    // Warp j owns rows 32j .. 32j+31 of every A stage. Per pass i (0..7) the warp
    // covers 4 rows x 128 B: lane -> row 32j + 4i + lane/8, physical 16-byte chunk
    // lane%8, which holds logical chunk (lane%8) ^ (row%8) under the swizzle.
    const int j = warp - kLnWarp0;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      const int m_blk = tile / p.n_blocks;
      float rstd[8], nmr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = m_blk * kBM + 32 * j + 4 * i + (lane >> 3);
        float2 st = make_float2(0.f, 0.f);
        if (row < p.M) st = p.stats[row];
        rstd[i] = st.y;
        nmr[i] = -st.x * st.y;
      }
      for (int kb = 0; kb < KB; ++kb) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bounded(&full[stage], phase, wc) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        mbar_try_wait(&full[stage], phase);  // completed: acquire for every lane
        uint8_t* a = sA + stage * kAStageBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 32 * j + 4 * i + (lane >> 3);
          const int pch = lane & 7;
          const int lch = pch ^ (r & 7);
          uint4* ptr = reinterpret_cast<uint4*>(a + r * 128 + pch * 16);
          const uint4 v = *ptr;
          const float4* g4 = reinterpret_cast<const float4*>(s_gamma + kb * kBK + lch * 8);
          const float4* b4 = reinterpret_cast<const float4*>(s_beta + kb * kBK + lch * 8);
          const float4 g0 = g4[0], g1 = g4[1], be0 = b4[0], be1 = b4[1];
          const float xs = rstd[i], xb = nmr[i];
          uint4 o;
          o.x = pack_bf16x2(fmaf(fmaf(bf16lo(v.x), xs, xb), g0.x, be0.x),
                            fmaf(fmaf(bf16hi(v.x), xs, xb), g0.y, be0.y));
          o.y = pack_bf16x2(fmaf(fmaf(bf16lo(v.y), xs, xb), g0.z, be0.z),
                            fmaf(fmaf(bf16hi(v.y), xs, xb), g0.w, be0.w));
          o.z = pack_bf16x2(fmaf(fmaf(bf16lo(v.z), xs, xb), g1.x, be1.x),
                            fmaf(fmaf(bf16hi(v.z), xs, xb), g1.y, be1.y));
          o.w = pack_bf16x2(fmaf(fmaf(bf16lo(v.w), xs, xb), g1.z, be1.z),
                            fmaf(fmaf(bf16hi(v.w), xs, xb), g1.w, be1.w));
          *ptr = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ LN statistics
// One warp per row: mean and 1/sqrt(biased var + eps), two passes over the row
// held in registers, reductions by warp shuffles.
template <int VPL>
__global__ void __launch_bounds__(256) ln_stats_kernel(const __nv_bfloat16* __restrict__ x, int M,
                                                       int C, float2* __restrict__ stats) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(row) * C);
  const int nvec = C >> 3;
  uint4 v[VPL];
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int idx = lane + 32 * i;
    v[i] = idx < nvec ? __ldg(xr + idx) : make_uint4(0, 0, 0, 0);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
    for (int e = 0; e < 4; ++e) sum += bf16lo(w[e]) + bf16hi(w[e]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / static_cast<float>(C);
  float sq = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (lane + 32 * i < nvec) {
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&v[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float d0 = bf16lo(w[e]) - mean, d1 = bf16hi(w[e]) - mean;
        sq = fmaf(d0, d0, sq);
        sq = fmaf(d1, d1, sq);
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (lane == 0) stats[row] = make_float2(mean, rsqrtf(sq / static_cast<float>(C) + kLnEps));
}

// ------------------------------------------------------------------ host launchers
template <int BN, bool LN_A, int EPI>
static cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const MlpParams& p,
                               int num_sms, cudaStream_t stream) {
  auto kern = mlp_gemm_kernel<BN, LN_A, EPI>;
  const size_t smem = mlp_smem_bytes(BN, LN_A, p.K);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  kern<<<grid, num_threads(LN_A), smem, stream>>>(tmA, tmB, p);
  return cudaGetLastError();
}

cudaError_t launch_ln_stats(const void* x, int M, int C, float* stats, cudaStream_t stream) {
  const int grid = (M + 7) / 8;
  const auto* xp = static_cast<const __nv_bfloat16*>(x);
  auto* sp = reinterpret_cast<float2*>(stats);
  if (C <= 256)
    ln_stats_kernel<1><<<grid, 256, 0, stream>>>(xp, M, C, sp);
  else if (C <= 512)
    ln_stats_kernel<2><<<grid, 256, 0, stream>>>(xp, M, C, sp);
  else if (C <= 1024)
    ln_stats_kernel<4><<<grid, 256, 0, stream>>>(xp, M, C, sp);
  else
    ln_stats_kernel<8><<<grid, 256, 0, stream>>>(xp, M, C, sp);
  return cudaGetLastError();
}

int fc1_block_n(int H) { return H % 256 == 0 ? 256 : (H % 128 == 0 ? 128 : 64); }
int fc2_block_n(int C) {
  return C % 256 == 0 ? 256 : (C % 192 == 0 ? 192 : (C % 128 == 0 ? 128 : 64));
}

cudaError_t launch_fc1(const CUtensorMap& tmX, const CUtensorMap& tmW1, const MlpParams& p, int bn,
                       int num_sms, cudaStream_t s) {
  switch (bn) {
    case 256: return launch_gemm<256, true, kEpiGelu>(tmX, tmW1, p, num_sms, s);
    case 128: return launch_gemm<128, true, kEpiGelu>(tmX, tmW1, p, num_sms, s);
    default: return launch_gemm<64, true, kEpiGelu>(tmX, tmW1, p, num_sms, s);
  }
}

cudaError_t launch_fc2(const CUtensorMap& tmHid, const CUtensorMap& tmW2, const MlpParams& p, int bn,
                       int num_sms, cudaStream_t s) {
  switch (bn) {
    case 256: return launch_gemm<256, false, kEpiResidShift>(tmHid, tmW2, p, num_sms, s);
    case 192: return launch_gemm<192, false, kEpiResidShift>(tmHid, tmW2, p, num_sms, s);
    case 128: return launch_gemm<128, false, kEpiResidShift>(tmHid, tmW2, p, num_sms, s);
    default: return launch_gemm<64, false, kEpiResidShift>(tmHid, tmW2, p, num_sms, s);
  }
}

}  // namespace rs
