// rs_mlp.cu -- the two contractions of the MLP sublayer (§3.3 Eq. (6) of
// "Representation Shift: Unifying Token Compression with FlashAttention") as
// persistent, warp-specialised tcgen05 GEMMs for sm_100a.
//
//   fc1 (folded LN, default):  z = rstd * (x' Wg^T - mean * G) + cb, a = GELU(z)
//        A = raw x' tiles (TMA); the LayerNorm is applied in the epilogue
//        through the fold of rs_ln.cu (Wg = W1 * gamma).
//   fc1 (staged LN):           a = GELU(LN(x') W1^T + b1); A = x' tiles (TMA)
//        normalised in place in shared memory by LN warps before the MMA.
//   fc2:  h = a W2^T + b2; y = x' + h;          A = a tiles (TMA)
//         P[r, j] = sum_{c in group j} (h - x')^2   -- Eq. (4) with D = L2, or with
//         the L1 and cosine distances of §3.3: sum |h - x'|, or the triple
//         (sum h x', sum h^2, sum x'^2) per column group
//
// One CTA per SM loops over 128 x BN output tiles (or a CTA pair over 256 x BN
// tiles, tcgen05 cta_group::2, for long reductions). Warp roles:
//   warp 0      TMA producer (A and B tiles, 64-wide K blocks, STAGES deep ring)
//   warp 1      TMEM owner and UMMA issuer (tcgen05.mma, M=128 or 256, N=BN, K=16)
//   warp 2      each tile's column vectors (16-warp epilogue only; otherwise the
//               producer loads them), warp 3 idle (the epilogue's first warp
//               sits on TMEM lane quadrant 0)
//   warps 4-11  epilogue (4-19 for the folded-LN fc1 at C <= 512): TMEM ->
//               registers -> LN fold / bias, GELU or residual/shift -> HBM through
//               per-warp TMA-store boxes
//   warps 12-15 (staged-LN fc1 only) LayerNorm staging of the A tile in place
// The fp32 accumulator is double-buffered in TMEM (2 x BN columns) so the
// epilogue of one tile overlaps the main loop of the next.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rs_internal.h"
#include "rs_gelu.cuh"
#include "rs_ptx.cuh"

namespace rs {

constexpr int kBM = 128;
constexpr int kBK = 64;                         // one 128-byte swizzle row of bf16
constexpr int kAStageBytes = kBM * kBK * 2;     // 16 KB
constexpr int kEpiWarp0 = 4;
constexpr int kLnWarp0 = 12;  // staged-LN kernel: after its 8 epilogue warps
constexpr int kNumLnWarps = 4;
constexpr int kSmemLimit = 232448;              // 227 KB opt-in per CTA
constexpr int kCtrlBytes = 512;                 // barriers, TMEM slot, abort flag
constexpr uint32_t kTmemCols = 512;

constexpr int kVecMaxBytes = 2 * 256 * 4;       // one tile's column vectors (fold: G and cb)

// One pipeline stage: the A tile (128 rows) and this CTA's rows of the B tile
// (all BN, or BN / 2 when a CTA pair shares the tile).
__host__ __device__ constexpr int stage_bytes(int bn, bool pair) {
  return kAStageBytes + (pair ? bn / 2 : bn) * kBK * 2;
}
// Per-tile column vectors the epilogue reads: the folded-LN G and cb (fp32) or
// the bias (bf16), for BN columns; double-buffered with the accumulator.
__host__ __device__ constexpr int vec_bytes(int bn, int epi) {
  return epi == kEpiGeluFold ? 2 * bn * 4 : bn * 2;
}
__host__ __device__ constexpr int vec_stride(int bn, int epi) {
  return (vec_bytes(bn, epi) + 127) / 128 * 128;
}
// The epilogue's per-warp output boxes (32 rows x out_box_cols bf16 each).
__host__ __device__ constexpr int out_bytes(int bn, int ew) {
  return ew * kEpiBoxRows * out_box_cols(bn, ew) * 2;
}
__host__ __device__ constexpr int fixed_smem(int bn, bool ln, int epi, int ew) {
  // alignment slack + control block + gamma/beta (bf16, up to RS_MAX_C each) +
  // the epilogue's per-warp output boxes + two tiles' column vectors
  return 1024 + kCtrlBytes + (ln ? 2 * RS_MAX_C * 2 : 0) + out_bytes(bn, ew) + 2 * kVecMaxBytes;
}
__host__ __device__ constexpr int num_stages(int bn, bool ln, int epi, bool pair, int ew) {
  return (kSmemLimit - fixed_smem(bn, ln, epi, ew)) / stage_bytes(bn, pair) > (pair ? 8 : 6)
             ? (pair ? 8 : 6)
             : (kSmemLimit - fixed_smem(bn, ln, epi, ew)) / stage_bytes(bn, pair);
}
// Epilogue warps EW: 8 (two per TMEM lane quadrant) or 16 (four). 16 pays off
// only where the epilogue's arithmetic rivals a short main loop (fc1 with
// C <= 512); the staged-LN kernel always uses 8 (its LN warps need registers).
__host__ __device__ constexpr int num_threads(bool ln, int ew) {
  return (kEpiWarp0 + ew + (ln ? kNumLnWarps : 0)) * 32;
}

size_t mlp_smem_bytes(int bn, bool ln, int epi, int K, int ew, bool pair) {
  return 1024 + static_cast<size_t>(num_stages(bn, ln, epi, pair, ew)) * stage_bytes(bn, pair) +
         out_bytes(bn, ew) + 2 * vec_stride(bn, epi) + kCtrlBytes +
         (ln ? 4 * static_cast<size_t>(K) : 0);
}

// Elementwise GELU with the same arithmetic as the fc1 epilogue (grid-stride,
// every lane of a warp stays active for the warp-uniform range choice).
__global__ void gelu_apply_kernel(const float* __restrict__ z, float* __restrict__ out, int n) {
  const int pairs = (n + 1) / 2;
  const int stride = gridDim.x * blockDim.x;
  const int iters = (pairs + stride - 1) / stride;
  for (int it = 0; it < iters; ++it) {
    const int pi = it * stride + blockIdx.x * blockDim.x + threadIdx.x;
    const int i = 2 * pi;
    const float z0 = i < n ? z[i] : 0.f;
    const float z1 = i + 1 < n ? z[i + 1] : 0.f;
    uint64_t zz[1] = {f2pack(z0, z1)}, gg[1];
    gelu2_block<1>(zz, gg);
    const float2 g = f2unpack(gg[0]);
    if (i < n) out[i] = g.x;
    if (i + 1 < n) out[i + 1] = g.y;
  }
}

cudaError_t launch_gelu(const float* z, float* out, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  int blocks = (pairs + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  gelu_apply_kernel<<<blocks, 256, 0, stream>>>(z, out, n);
  return cudaGetLastError();
}

template <int BN, bool LN_A, int EPI, int EW, bool PAIR>
__global__ void __launch_bounds__(num_threads(LN_A, EW), 1)
    mlp_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmOut, const MlpParams p) {
  static_assert(!(PAIR && LN_A), "the staged-LN kernel runs on single CTAs");
  constexpr int kBRows = PAIR ? BN / 2 : BN;       // rows of the B tile this CTA loads
  constexpr int kBStageBytes = kBRows * kBK * 2;
  constexpr int STAGES = num_stages(BN, LN_A, EPI, PAIR, EW);
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;      // output rows of one tile
  constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, BN);
  // bytes that complete one stage's full barrier (the leader's, for a pair)
  constexpr uint32_t kTxBytes = (PAIR ? 2 : 1) * (kAStageBytes + kBStageBytes);
  constexpr int kNumEpiWarps = EW;
  static_assert(EW == 8 || EW == 16, "epilogue warps");
  static_assert(!LN_A || EW == 8, "staged-LN kernel: 8 epilogue warps");
  constexpr int kOutBytes = out_bytes(BN, EW);
  constexpr int kVecBytes = vec_bytes(BN, EPI);
  constexpr int kVecStride = vec_stride(BN, EPI);
  static_assert(BN % 64 == 0 && BN <= 256, "BN");
  static_assert(2 * BN <= static_cast<int>(kTmemCols), "TMEM double buffer");
  static_assert(STAGES >= 2, "pipeline depth");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kAStageBytes;
  uint8_t* sOut = sB + STAGES * kBStageBytes;
  uint8_t* sVec = sOut + kOutBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sVec + 2 * kVecStride);
  uint64_t* empty = full + STAGES;
  uint64_t* aready = empty + STAGES;
  uint64_t* tfull = aready + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* vfull = tempty + 2;
  uint64_t* vempty = vfull + 2;
  uint64_t* drain = vempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __nv_bfloat16* s_gamma =
      reinterpret_cast<__nv_bfloat16*>(sVec + 2 * kVecStride + kCtrlBytes);
  __nv_bfloat16* s_beta = s_gamma + p.K;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB = p.K / kBK;
  // A CTA pair (a cluster of two) shares each tile: CTA `rank` holds A rows
  // 128 * rank .. +127 of the 256-row tile and B rows BN/2 * rank .. +BN/2-1; the
  // leader (rank 0) issues the MMAs, whose accumulator rows land in the TMEM of
  // the CTA that holds them.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&aready[s], kNumLnWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 2 * kNumEpiWarps : kNumEpiWarps);
      mbar_init(&vfull[a], 1);
      mbar_init(&vempty[a], kNumEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  // Nothing above touched global memory: let the next kernel launch, then wait
  // for the previous one to finish before reading anything it may have written.
  pdl_trigger();
  pdl_wait();
  if constexpr (LN_A) {
    const uint4* g = reinterpret_cast<const uint4*>(p.ln_gamma);
    const uint4* b = reinterpret_cast<const uint4*>(p.ln_beta);
    for (int i = threadIdx.x; i < p.K / 8; i += blockDim.x) {
      reinterpret_cast<uint4*>(s_gamma)[i] = __ldg(g + i);
      reinterpret_cast<uint4*>(s_beta)[i] = __ldg(b + i);
    }
  }
  tc_fence_before_sync();
  if constexpr (PAIR) {
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};

  // A tile's column vectors (the bias, or the LN fold's G and cb) go into the
  // buffer of the accumulator it will use once the epilogue is done with that
  // buffer's previous tile. The producer loads them at each tile's start, except
  // with the 16-warp epilogue (short reductions): there the producer runs a whole
  // tile ahead of that release, so warp 2 loads them and the operand stream never
  // waits on the epilogue.
  constexpr bool kVecWarp = EW == 16;
  int vacc = 0;
  uint32_t vphase = 0;
  int vpend0 = -1, vpend1 = -1;
  auto load_vectors = [&](int n_blk) -> bool {
    if (!wait_bounded(&vempty[vacc], vphase ^ 1u, wc)) return false;
    mbar_arrive_expect_tx(&vfull[vacc], kVecBytes);
    uint8_t* vdst = sVec + vacc * kVecStride;
    if constexpr (EPI == kEpiGeluFold) {
      bulk_load(vdst, p.colG + n_blk * BN, BN * 4, &vfull[vacc]);
      bulk_load(vdst + BN * 4, p.colC + n_blk * BN, BN * 4, &vfull[vacc]);
    } else {
      bulk_load(vdst, p.bias + n_blk * BN, BN * 2, &vfull[vacc]);
    }
    if (vacc == 0) vpend0 = static_cast<int>(vphase); else vpend1 = static_cast<int>(vphase);
    if (++vacc == 2) { vacc = 0; vphase ^= 1u; }
    return true;
  };
  // Every vector copy this thread issued must land before the CTA may exit.
  auto finish_vectors = [&]() {
    if (vpend0 >= 0) wait_bounded(&vfull[0], static_cast<uint32_t>(vpend0), wc, false);
    if (vpend1 >= 0) wait_bounded(&vfull[1], static_cast<uint32_t>(vpend1), wc, false);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      // stages with a copy in flight (bit s) and the phase it completes (bit s)
      uint32_t pend_mask = 0, pend_phase = 0;
      // both CTAs' loads of a pair complete on the leader's full barriers
      const uint32_t full_leader = PAIR ? mapa_shared(smem_u32(&full[0]), 0u) : 0u;
      for (int tile = unit0; tile < p.num_tiles; tile += units) {
        const int m_blk = tile / p.n_blocks, n_blk = tile % p.n_blocks;
        if constexpr (!kVecWarp) {
          if (!load_vectors(n_blk)) break;
        }
        // test hook: leave one stage unfilled so the consumer's wait runs out
        const int skip_kb = (blockIdx.x == 0 && tile == unit0) ? p.debug_skip_kb : -1;
        const int a_row = m_blk * kTileM + static_cast<int>(rank) * kBM;
        const int b_row = n_blk * BN + static_cast<int>(rank) * kBRows;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, wc)) { ok = false; break; }
          if (kb != skip_kb) {
            if (leader) mbar_arrive_expect_tx(&full[stage], kTxBytes);
            if constexpr (PAIR) {
              const uint32_t fb = full_leader + static_cast<uint32_t>(stage) * 8u;
              tma_load_2d_pair(sA + stage * kAStageBytes, &tmA, fb, kb * kBK, a_row);
              tma_load_2d_pair(sB + stage * kBStageBytes, &tmB, fb, kb * kBK, b_row);
            } else {
              tma_load_2d(sA + stage * kAStageBytes, &tmA, &full[stage], kb * kBK, a_row);
              tma_load_2d(sB + stage * kBStageBytes, &tmB, &full[stage], kb * kBK, b_row);
            }
            const uint32_t bit = 1u << stage;
            pend_mask |= bit;
            pend_phase = (pend_phase & ~bit) | (phase << stage);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // Every copy this thread issued must land before the CTA may exit (on a
      // pair the non-leader's copies complete on the leader's barriers, which the
      // leader waits for).
      if (leader) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s)
          if (pend_mask & (1u << s)) wait_bounded(&full[s], (pend_phase >> s) & 1u, wc, false);
      }
      if constexpr (!kVecWarp) finish_vectors();
      if constexpr (PAIR) {
        // The leader's releases of every stage (multicast commits into this CTA's
        // empty barriers) have all arrived before the CTA may exit.
        for (int i = 0; i < STAGES; ++i) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, wc)) break;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (kVecWarp && warp == 2) {
    // ------------------------------------------------------------ column vectors
    if (lane == 0) {
      for (int tile = unit0; tile < p.num_tiles; tile += units)
        if (!load_vectors(tile % p.n_blocks)) break;
      finish_vectors();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued = false;
      for (int tile = unit0; tile < p.num_tiles; tile += units) {
        // a pair's tempty also counts the peer's epilogue warps (remote arrivals)
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, wc, true, PAIR)) break;
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
          for (int k = 0; k < kBK / 16; ++k) {
            if constexpr (PAIR)
              umma_bf16_pair(d_tmem, ad + 2u * k, bd + 2u * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
            else
              umma_bf16(d_tmem, ad + 2u * k, bd + 2u * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          issued = true;
          if constexpr (PAIR)
            umma_commit_pair_mc(&empty[stage], 0x3);  // both CTAs' producers
          else
            umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR)
          umma_commit_pair_mc(&tfull[acc], 0x3);  // both CTAs' epilogues
        else
          umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (*abort_flag && issued) {
        // Drain: wait until every MMA issued so far has finished with TMEM and smem.
        if constexpr (PAIR)
          umma_commit_pair(drain);
        else
          umma_commit(drain);
        wait_bounded(drain, 0u, wc, false);
      }
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kNumEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // Warp -> TMEM lane quadrant q (rows 32q..32q+31 of the tile) and one of
    // kNumEpiWarps/4 column groups of the BN columns, in 16-column chunks: the
    // TMEM load (and for fc2 the residual row slice) of chunk n+1 is in flight
    // while chunk n is processed. The accumulator goes back to the MMA warp as
    // soon as its last chunk is in registers. The chunks fill the warp's output
    // box (32 rows x kBoxCols columns, 16 or 32: the 32- or 64-byte swizzle, 16-byte
    // unit j of row r at j ^ ((r >> 2) & 1) or j ^ ((r >> 1) & 3)), which leaves by one
    // TMA store when full; rows past M are clipped by the store.
    constexpr int kGroups = kNumEpiWarps / 4;
    constexpr int kCols = BN / kGroups;  // columns of one warp
    constexpr int NCH = kCols / kEpiChunkCols;
    constexpr int kBoxCols = out_box_cols(BN, EW);
    constexpr int CPB = kBoxCols / kEpiChunkCols;  // chunks per box
    constexpr int kBoxBytes = kEpiBoxRows * kBoxCols * 2;
    static_assert(kCols % kBoxCols == 0 && kBoxCols % kEpiChunkCols == 0, "chunking");
    static_assert(kBoxCols == 16 || kBoxCols == 32, "box swizzle");
    const int q = warp & 3;
    const int grp = (warp - kEpiWarp0) >> 2;
    uint8_t* box = sOut + (warp - kEpiWarp0) * kBoxBytes;
    const uint32_t box_u32 = smem_u32(box);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = unit0; tile < p.num_tiles; tile += units) {
      const int m_blk = tile / p.n_blocks, n_blk = tile % p.n_blocks;
      const int row0 = m_blk * kTileM + static_cast<int>(rank) * kBM;  // this CTA's first row
      int ok = 1;
      if (lane == 0)
        ok = (wait_bounded(&vfull[acc], acc_phase, wc) && wait_bounded(&tfull[acc], acc_phase, wc))
                 ? 1
                 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      mbar_try_wait(&vfull[acc], acc_phase);  // completed: acquire for every lane
      mbar_try_wait(&tfull[acc], acc_phase);
      tc_fence_after_sync();
      const int row = row0 + q * 32 + lane;
      const bool row_ok = row < p.M;
      const bool box_live = row0 + q * 32 < p.M;  // the warp's box holds rows of the output
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + grp * kCols);
      const int col0 = n_blk * BN + grp * kCols;
      const uint32_t vec_u32 = smem_u32(sVec + acc * kVecStride);
      float part = 0.f;                      // L2: sum (h - x')^2; L1: sum |h - x'|
      float c_hx = 0.f, c_hh = 0.f, c_xx = 0.f;  // cosine: sum h x', sum h^2, sum x'^2
      uint64_t nmu2 = 0, rs2 = 0;  // folded LN: (-mean, -mean), (rstd, rstd) of this row
      if constexpr (EPI == kEpiGeluFold) {
        float2 st = make_float2(0.f, 0.f);
        if (row_ok) st = p.stats[row];
        nmu2 = f2pack(-st.x, -st.x);
        rs2 = f2pack(st.y, st.y);
      }
      const uint4* xrow =
          reinterpret_cast<const uint4*>(p.resid + static_cast<size_t>(row) * p.N + col0);
      // whole-block shift (§3.3 case (iii)): the distance compares y = x' + h with
      // the block input at p.shift_ref instead of h with x'
      const bool has_ref = EPI == kEpiResidShift && p.shift_ref != nullptr;
      const uint4* zrow =
          reinterpret_cast<const uint4*>(p.shift_ref + static_cast<size_t>(row) * p.N + col0);
      uint32_t ra[16], rb[16];
      uint4 xa[2] = {}, xb[2] = {}, za[2] = {}, zb[2] = {};
      tmem_ld16_async(t_row, ra);
      if constexpr (EPI == kEpiResidShift) {
        if (row_ok) {
          xa[0] = __ldg(xrow);
          xa[1] = __ldg(xrow + 1);
          if (has_ref) {
            za[0] = __ldg(zrow);
            za[1] = __ldg(zrow + 1);
          }
        }
      }
#pragma unroll
      for (int n = 0; n < NCH; ++n) {
        uint32_t(&r)[16] = (n & 1) ? rb : ra;
        uint32_t(&nx)[16] = (n & 1) ? ra : rb;
        uint4(&xv)[2] = (n & 1) ? xb : xa;
        uint4(&xn)[2] = (n & 1) ? xa : xb;
        uint4(&zv)[2] = (n & 1) ? zb : za;
        uint4(&zn)[2] = (n & 1) ? za : zb;
        tmem_wait_ld();
        reg_fence16(r);
        if (n + 1 < NCH) {
          tmem_ld16_async(t_row + (n + 1) * 16, nx);
          if constexpr (EPI == kEpiResidShift) {
            if (row_ok) {
              xn[0] = __ldg(xrow + (n + 1) * 2);
              xn[1] = __ldg(xrow + (n + 1) * 2 + 1);
              if (has_ref) {
                zn[0] = __ldg(zrow + (n + 1) * 2);
                zn[1] = __ldg(zrow + (n + 1) * 2 + 1);
              }
            }
          }
        } else {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if (PAIR && !leader)
              mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0u));
            else
              mbar_arrive(&tempty[acc]);
          }
        }
        const int c = n * 16;
        const uint32_t cvec = grp * kCols + c;  // column of this chunk within the tile
        uint32_t outw[8];
        if constexpr (EPI == kEpiGeluFold) {
          // z = rstd * (acc - mean * G[col]) + cb[col], two columns per step
          uint64_t z2[8], g2[8];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 g4 = lds128(vec_u32 + (cvec + 4 * v) * 4);
            const uint4 c4 = lds128(vec_u32 + BN * 4 + (cvec + 4 * v) * 4);
            const uint64_t ga = (static_cast<uint64_t>(g4.y) << 32) | g4.x;
            const uint64_t gb = (static_cast<uint64_t>(g4.w) << 32) | g4.z;
            const uint64_t ca = (static_cast<uint64_t>(c4.y) << 32) | c4.x;
            const uint64_t cb = (static_cast<uint64_t>(c4.w) << 32) | c4.z;
            z2[2 * v] = ffma2(
                rs2, ffma2(nmu2, ga, f2pack(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]))),
                ca);
            z2[2 * v + 1] = ffma2(
                rs2,
                ffma2(nmu2, gb, f2pack(__uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]))),
                cb);
          }
          if (!p.linear) {
            gelu2_block<8>(z2, g2);
          } else {  // no activation: the attention sublayer's QKV projection
#pragma unroll
            for (int e = 0; e < 8; ++e) g2[e] = z2[e];
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 g = f2unpack(g2[e]);
            outw[e] = pack_bf16x2(g.x, g.y);
          }
        } else {
          uint32_t bw[8];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const uint4 b4 = lds128(vec_u32 + (cvec + 8 * v) * 2);
            bw[4 * v] = b4.x;
            bw[4 * v + 1] = b4.y;
            bw[4 * v + 2] = b4.z;
            bw[4 * v + 3] = b4.w;
          }
          if constexpr (EPI == kEpiGelu) {
            uint64_t z2[8], g2[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              z2[e] = f2pack(__uint_as_float(r[2 * e]) + bf16lo(bw[e]),
                             __uint_as_float(r[2 * e + 1]) + bf16hi(bw[e]));
            gelu2_block<8>(z2, g2);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 g = f2unpack(g2[e]);
              outw[e] = pack_bf16x2(g.x, g.y);
            }
          } else {
            const uint32_t* xw = reinterpret_cast<const uint32_t*>(xv);
            const uint32_t* zw = reinterpret_cast<const uint32_t*>(zv);
            // h in fp32 before rounding; the distance compares (f, g) = (h, x') or, for
            // the whole-block shift, (x' + h, block input). Uniform over the launch.
#define RS_SHIFT_OPERANDS(e)                                              \
  const float x0 = bf16lo(xw[e]), x1 = bf16hi(xw[e]);                     \
  const float h0 = __uint_as_float(r[2 * (e)]) + bf16lo(bw[e]);           \
  const float h1 = __uint_as_float(r[2 * (e) + 1]) + bf16hi(bw[e]);       \
  outw[e] = pack_bf16x2(x0 + h0, x1 + h1);                                \
  const float f0 = has_ref ? x0 + h0 : h0, f1 = has_ref ? x1 + h1 : h1;   \
  const float g0 = has_ref ? bf16lo(zw[e]) : x0, g1 = has_ref ? bf16hi(zw[e]) : x1;
            if (p.dist == kDistCos) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                RS_SHIFT_OPERANDS(e)
                c_hx = fmaf(f0, g0, c_hx);
                c_hx = fmaf(f1, g1, c_hx);
                c_hh = fmaf(f0, f0, c_hh);
                c_hh = fmaf(f1, f1, c_hh);
                c_xx = fmaf(g0, g0, c_xx);
                c_xx = fmaf(g1, g1, c_xx);
              }
            } else if (p.dist == kDistL1) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                RS_SHIFT_OPERANDS(e)
                part += fabsf(f0 - g0);
                part += fabsf(f1 - g1);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                RS_SHIFT_OPERANDS(e)
                const float d0 = f0 - g0, d1 = f1 - g1;
                part = fmaf(d0, d0, part);
                part = fmaf(d1, d1, part);
              }
            }
#undef RS_SHIFT_OPERANDS
          }
        }
        if (n + 1 == NCH) {
          // the last chunk's column vectors are read: the buffer may be refilled
          __syncwarp();
          if (lane == 0) mbar_arrive(&vempty[acc]);
        }
        if (n % CPB == 0) {
          // the box's previous store has read it before it is written again
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
        }
        {
          const uint32_t u0 = static_cast<uint32_t>((n % CPB) * 2);  // 16-byte units of the chunk
          const uint32_t sw = kBoxCols == 16 ? (lane >> 2) & 1 : (lane >> 1) & 3;
          sts128(box_u32 + lane * (kBoxCols * 2) + ((u0 ^ sw) << 4),
                 make_uint4(outw[0], outw[1], outw[2], outw[3]));
          sts128(box_u32 + lane * (kBoxCols * 2) + (((u0 + 1) ^ sw) << 4),
                 make_uint4(outw[4], outw[5], outw[6], outw[7]));
        }
        if (n % CPB == CPB - 1) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && box_live) {
            tma_store_2d(&tmOut, box, col0 + c - (CPB - 1) * kEpiChunkCols, row0 + q * 32);
            bulk_commit_group();
          }
        }
      }
      if constexpr (EPI == kEpiResidShift) {
        if (row_ok) {
          float* pr = p.partials + static_cast<size_t>(row) * p.num_partials;
          const int g = n_blk * kGroups + grp;  // column group of the row
          if (p.dist == kDistCos) {
            pr[3 * g] = c_hx;
            pr[3 * g + 1] = c_hh;
            pr[3 * g + 2] = c_xx;
          } else {
            pr[g] = part;
          }
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  } else if (LN_A && warp >= kLnWarp0) {
    // ------------------------------------------------------------ LayerNorm staging
    // The A stage holds raw x' (TMA, 128-byte swizzle: 16-byte chunk c of row r
    // at physical chunk c ^ (r % 8)). Warp j normalises rows 32j .. 32j+31 in
    // place. Lane l always handles logical chunk c = l % 8 (columns 8c .. 8c+7 of
    // the k-block) of rows 32j + 4i + l/8, i = 0..7, so its gamma/beta slice is
    // read once per stage and every shared access is conflict-free.
    const int j = warp - kLnWarp0;
    const int c = lane & 7;
    const int rsub = lane >> 3;
    const uint32_t sA_u32 = smem_u32(sA);
    const uint32_t g_u32 = smem_u32(s_gamma) + c * 16;
    const uint32_t b_u32 = smem_u32(s_beta) + c * 16;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = unit0; tile < p.num_tiles && ok; tile += units) {
      const int m_blk = tile / p.n_blocks;
      uint64_t rs2[8], nm2[8];  // (rstd, rstd) and (-mean*rstd, -mean*rstd) per row
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = m_blk * kBM + 32 * j + 4 * i + rsub;
        float2 st = make_float2(0.f, 0.f);
        if (row < p.M) st = p.stats[row];
        rs2[i] = f2pack(st.y, st.y);
        nm2[i] = f2pack(-st.x * st.y, -st.x * st.y);
      }
      for (int kb = 0; kb < KB; ++kb) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bounded(&full[stage], phase, wc) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) { ok = false; break; }
        mbar_try_wait(&full[stage], phase);  // completed: acquire for every lane
        const uint4 gq = lds128(g_u32 + kb * 128);
        const uint4 bq = lds128(b_u32 + kb * 128);
        const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
        const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w};
        uint64_t g2[4], b2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          g2[e] = f2pack(bf16lo(gw[e]), bf16hi(gw[e]));
          b2[e] = f2pack(bf16lo(bw[e]), bf16hi(bw[e]));
        }
        const uint32_t a_u32 = sA_u32 + stage * kAStageBytes;
        uint32_t addr[8];
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 32 * j + 4 * i + rsub;
          addr[i] = a_u32 + r * 128 + ((c ^ (r & 7)) << 4);
          v[i] = lds128(addr[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t xw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint64_t x2 = f2pack(bf16lo(xw[e]), bf16hi(xw[e]));
            const float2 u = f2unpack(ffma2(ffma2(x2, rs2[i], nm2[i]), g2[e], b2[e]));
            o[e] = pack_bf16x2(u.x, u.y);
          }
          sts128(addr[i], make_uint4(o[0], o[1], o[2], o[3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aready[stage]);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  }

  __syncthreads();
  if constexpr (PAIR) {
    // After an abort a CTA may still have loads in flight that complete on the
    // other CTA's barriers and that neither CTA can wait for: give them time to
    // land. Then neither CTA leaves (or frees TMEM) before the other is done.
    if (threadIdx.x == 0 && (*abort_flag || *reinterpret_cast<volatile int*>(p.err) != 0))
      spin_ns(1000000);
    cluster_sync();
  }
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem_base, kTmemCols);
    else
      tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ host launchers
template <int BN, bool LN_A, int EPI, int EW = 8, bool PAIR = false>
static cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB,
                               const CUtensorMap& tmOut, const MlpParams& p, int num_sms,
                               cudaStream_t stream, bool pdl) {
  auto kern = mlp_gemm_kernel<BN, LN_A, EPI, EW, PAIR>;
  const size_t smem = mlp_smem_bytes(BN, LN_A, EPI, p.K, EW, PAIR);
  const int threads = num_threads(LN_A, EW);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if constexpr (PAIR) {
    // One CTA pair per two SMs, as many pairs as can be resident at once (an SM
    // whose partner in its GPC is missing stays idle).
    static const int max_pairs = [&]() {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (num_sms / 2));
      cfg.blockDim = dim3(threads);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms / 2;
      }
      return n < num_sms / 2 ? n : num_sms / 2;
    }();
    const int pairs = p.num_tiles < max_pairs ? p.num_tiles : max_pairs;
    return launch_cluster(kern, 2 * pairs, threads, smem, stream, pdl, 2, tmA, tmB, tmOut, p);
  } else {
    const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
    return launch(kern, grid, threads, smem, stream, pdl, tmA, tmB, tmOut, p);
  }
}

int fc1_block_n(int H) { return H % 256 == 0 ? 256 : (H % 128 == 0 ? 128 : 64); }
int fc2_block_n(int C) {
  return C % 256 == 0 ? 256 : (C % 192 == 0 ? 192 : (C % 128 == 0 ? 128 : 64));
}

template <int BN, int EW>
static cudaError_t launch_fold(const CUtensorMap& tmX, const CUtensorMap& tmW1,
                               const CUtensorMap& tmHid, const MlpParams& p, bool pair,
                               int num_sms, cudaStream_t s, bool pdl) {
  return pair ? launch_gemm<BN, false, kEpiGeluFold, EW, true>(tmX, tmW1, tmHid, p, num_sms, s, pdl)
              : launch_gemm<BN, false, kEpiGeluFold, EW, false>(tmX, tmW1, tmHid, p, num_sms, s,
                                                                  pdl);
}

cudaError_t launch_fc1(const CUtensorMap& tmX, const CUtensorMap& tmW1, const CUtensorMap& tmHid,
                       const MlpParams& p, int bn, bool staged_ln, bool pair, int num_sms,
                       cudaStream_t s, bool pdl) {
  if (staged_ln) {
    if (pair) return cudaErrorInvalidValue;
    switch (bn) {
      case 256: return launch_gemm<256, true, kEpiGelu>(tmX, tmW1, tmHid, p, num_sms, s, pdl);
      case 128: return launch_gemm<128, true, kEpiGelu>(tmX, tmW1, tmHid, p, num_sms, s, pdl);
      default: return launch_gemm<64, true, kEpiGelu>(tmX, tmW1, tmHid, p, num_sms, s, pdl);
    }
  }
  if (gemm_epi_warps(true, p.K) == 16) {
    switch (bn) {
      case 256: return launch_fold<256, 16>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
      case 128: return launch_fold<128, 16>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
      default: return launch_fold<64, 16>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
    }
  }
  switch (bn) {
    case 256: return launch_fold<256, 8>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
    case 128: return launch_fold<128, 8>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
    default: return launch_fold<64, 8>(tmX, tmW1, tmHid, p, pair, num_sms, s, pdl);
  }
}

template <int BN>
static cudaError_t launch_resid(const CUtensorMap& tmHid, const CUtensorMap& tmW2,
                                const CUtensorMap& tmY, const MlpParams& p, bool pair, int num_sms,
                                cudaStream_t s, bool pdl) {
  return pair ? launch_gemm<BN, false, kEpiResidShift, 8, true>(tmHid, tmW2, tmY, p, num_sms, s, pdl)
              : launch_gemm<BN, false, kEpiResidShift, 8, false>(tmHid, tmW2, tmY, p, num_sms, s,
                                                                   pdl);
}

cudaError_t launch_fc2(const CUtensorMap& tmHid, const CUtensorMap& tmW2, const CUtensorMap& tmY,
                       const MlpParams& p, int bn, bool pair, int num_sms, cudaStream_t s,
                       bool pdl) {
  switch (bn) {
    case 256: return launch_resid<256>(tmHid, tmW2, tmY, p, pair, num_sms, s, pdl);
    case 192: return launch_resid<192>(tmHid, tmW2, tmY, p, pair, num_sms, s, pdl);
    case 128: return launch_resid<128>(tmHid, tmW2, tmY, p, pair, num_sms, s, pdl);
    default: return launch_resid<64>(tmHid, tmW2, tmY, p, pair, num_sms, s, pdl);
  }
}

}  // namespace rs
