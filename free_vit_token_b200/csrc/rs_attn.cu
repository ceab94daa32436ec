// rs_attn.cu -- the attention core of the ViT attention sublayer on sm_100a:
// per sample and head, O = Softmax(Q K^T / sqrt(d)) V (Eq. (1) of
// "Representation Shift: Unifying Token Compression with FlashAttention", one
// head of width d = 64), without materialising the L x L score matrix.
//
// One CTA owns 128 queries of one (sample, head) and walks the keys in blocks
// of 64 (online softmax); three CTAs share an SM (128 TMEM columns and ~65 KB of
// shared memory each), so one CTA's softmax overlaps the others' loads and MMAs:
//   warp 0      TMA producer: the Q tile once, then the K and V tiles of each key
//               block into two-stage rings of their own (3-D tensor maps over
//               [B, L, 3C], so rows past a sample's L read as zero and never cross
//               samples). A K stage is free once its S MMA has finished and a V
//               stage once its P V MMA has, so K_{j+2} is on its way while block j's
//               softmax runs and neither ring waits on the other;
//   warp 1      owns the CTA's TMEM columns and issues the MMAs:
//               S_j = Q K_j^T (M = 128, N = 64, K = 64) into the TMEM score
//               buffer, and O += P_j V_j (M = 128, N = 64, K = 64, V read MN-major)
//               into the TMEM output accumulator;
//   warps 2..5  softmax, one query row per thread (its TMEM lane): row maximum
//               over the block, P = 2^(S log2(e)/sqrt(d) - m_ref) rounded to bf16
//               into shared memory (the A operand of P V, 128-byte swizzle) and
//               the running sum l. The reference maximum m_ref moves, and O (in
//               TMEM) and l are rescaled by 2^(m_ref - m_new), only when a row's
//               maximum grows by more than 8 (P then stays below 2^8, exact in the
//               arithmetic that follows); at the end O / l goes out as bf16.
// S is read out of TMEM at the start of a block, so S_{j+1} is computed while
// the softmax of block j proceeds, and P V of block j runs while block j+1's
// exponentials are computed. Every wait is bounded (timeout -> error flag, CTA
// abort, drain, TMEM freed).
#include <cstdint>

#include "rs_internal.h"
#include "rs_ptx.cuh"

namespace rs {

namespace {

constexpr int kHd = 64;                         // head width d
constexpr int kQRows = 128;                     // queries per CTA (TMEM lanes)
constexpr int kKeys = 64;                       // keys per block
constexpr int kKvStages = 2;
constexpr int kBox = kQRows * kHd * 2;          // the Q tile: 128 rows x 64 columns (16 KB)
constexpr int kKvBox = kKeys * kHd * 2;         // a K or V tile: 64 rows x 64 columns (8 KB)
constexpr int kPBytes = kQRows * kKeys * 2;     // P: 128 rows x 64 keys (16 KB)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kTmemO = kKeys;              // O after the score buffer
constexpr int kCtrl = 256;
constexpr float kRescaleAbove = 8.f;            // log2 of the largest P kept unrescaled

constexpr int smem_bytes() {
  return 1024 + kBox + kKvStages * 2 * kKvBox + kPBytes + kCtrl;
}

__global__ void __launch_bounds__(kThreads, 3)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmKV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kBox;                       // stage s: K at sK + 2 kKvBox s, V after it
  uint8_t* sP = sK + kKvStages * 2 * kKvBox;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sP + kPBytes);
  uint64_t* k_full = q_full + 1;
  uint64_t* v_full = k_full + kKvStages;
  uint64_t* k_empty = v_full + kKvStages;
  uint64_t* v_empty = k_empty + kKvStages;
  uint64_t* s_full = v_empty + kKvStages;
  uint64_t* s_empty = s_full + 1;
  uint64_t* p_full = s_empty + 1;
  uint64_t* pv_full = p_full + 1;
  uint64_t* drain = pv_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto sKs = [&](int s) { return sK + s * 2 * kKvBox; };
  auto sVs = [&](int s) { return sK + s * 2 * kKvBox + kKvBox; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQRows;
  const int head = blockIdx.y;
  const int b = blockIdx.z;
  const int nkb = (p.L + kKeys - 1) / kKeys;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int C = p.C;
      mbar_arrive_expect_tx(q_full, kBox);
      tma_load_3d(sQ, &tmQ, q_full, head * kHd, q0, b);
      int k_issued = 0, v_issued = 0;
      const bool hook = blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
      // K_j, then V_{j-1}: the S MMA of a block comes before its P V MMA
      for (int j = 0; j <= nkb; ++j) {
        if (j < nkb) {
          const int s = j % kKvStages;
          if (j >= kKvStages && !wait_bounded(&k_empty[s], ((j / kKvStages) - 1) & 1, wc)) break;
          // test hook: stop loading, so that the MMA warp's wait for this block runs out
          if (hook && j == p.debug_skip_block) break;
          mbar_arrive_expect_tx(&k_full[s], kKvBox);
          tma_load_3d(sKs(s), &tmKV, &k_full[s], C + head * kHd, j * kKeys, b);
          k_issued = j + 1;
        }
        if (j >= 1) {
          const int i = j - 1, s = i % kKvStages;
          if (i >= kKvStages && !wait_bounded(&v_empty[s], ((i / kKvStages) - 1) & 1, wc)) break;
          mbar_arrive_expect_tx(&v_full[s], kKvBox);
          tma_load_3d(sVs(s), &tmKV, &v_full[s], 2 * C + head * kHd, i * kKeys, b);
          v_issued = i + 1;
        }
      }
      // every load issued has landed before the CTA may finish (after an abort too)
      wait_bounded(q_full, 0u, wc, false);
      for (int j = k_issued > kKvStages ? k_issued - kKvStages : 0; j < k_issued; ++j)
        wait_bounded(&k_full[j % kKvStages], (j / kKvStages) & 1, wc, false);
      for (int j = v_issued > kKvStages ? v_issued - kKvStages : 0; j < v_issued; ++j)
        wait_bounded(&v_full[j % kKvStages], (j / kKvStages) & 1, wc, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kQRows, kKeys);
      constexpr uint32_t kIdO = idesc_bf16_f32_bmn(kQRows, kHd);
      const uint32_t q_u32 = smem_u32(sQ);
      const uint32_t p_u32 = smem_u32(sP);
      auto issue_pv = [&](int i) -> bool {
        const int st = i % kKvStages;
        if (!wait_bounded(p_full, i & 1, wc)) return false;
        if (!wait_bounded(&v_full[st], (i / kKvStages) & 1, wc)) return false;
        tc_fence_after_sync();
        const uint32_t v_u32 = smem_u32(sVs(st));
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          umma_bf16(tmem + kTmemO, sw128_kmajor_desc(p_u32) + kk * 2,
                    sw128_mnmajor_desc(v_u32 + kk * 2048, kKvBox), kIdO,
                    (i > 0 || kk > 0) ? 1u : 0u);
        umma_commit(pv_full);
        umma_commit(&v_empty[st]);
        return true;
      };
      bool ok = wait_bounded(q_full, 0u, wc);
      for (int j = 0; ok && j < nkb; ++j) {
        const int st = j % kKvStages;
        if (!wait_bounded(&k_full[st], (j / kKvStages) & 1, wc) ||
            (j >= 1 && !wait_bounded(s_empty, (j - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t k_u32 = smem_u32(sKs(st));
#pragma unroll
        for (int kk = 0; kk < kHd / 16; ++kk)
          umma_bf16(tmem, sw128_kmajor_desc(q_u32) + kk * 2, sw128_kmajor_desc(k_u32) + kk * 2,
                    kIdS, kk > 0 ? 1u : 0u);
        umma_commit(s_full);
        umma_commit(&k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) ok = false;
      }
      if (ok) issue_pv(nkb - 1);
      // drain: every MMA issued has finished with TMEM and shared memory
      umma_commit(drain);
      wait_bounded(drain, 0u, wc, false);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3;                    // TMEM lane quadrant of this warp
    const int r = qd * 32 + lane;               // query row within the tile
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float c = 1.4426950408889634f / 8.f;  // log2(e) / sqrt(64)
    float m = -INFINITY;                        // reference maximum, in log2 units
    float l = 0.f;                              // running sum of P
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(bar, parity, wc) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) mbar_try_wait(bar, parity);  // completed: acquire for every lane
      return ok != 0;
    };
    const uint32_t p_row = smem_u32(sP) + r * 128;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      if (!wait_all(s_full, j & 1)) { ok = false; break; }
      tc_fence_after_sync();
      // the block's 64 scores of this row, keys past the sample's end set to -inf
      uint32_t a0[32], a1[32];
      tmem_ld32_async(t_lane, a0);
      tmem_ld32_async(t_lane + 32, a1);
      tmem_wait_ld();
      reg_fence(a0);
      reg_fence(a1);
      // the score buffer is read: the MMA warp may compute the next block's scores
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      const int kvalid = p.L - j * kKeys;       // keys of this block inside the sample (>= 1)
      if (kvalid < kKeys) {  // the last block of a ragged sequence (warp-uniform)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          if (e >= kvalid) a0[e] = __float_as_uint(-INFINITY);
          if (32 + e >= kvalid) a1[e] = __float_as_uint(-INFINITY);
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        mx0 = fmaxf(mx0, __uint_as_float(a0[e]));
        mx1 = fmaxf(mx1, __uint_as_float(a1[e]));
      }
      const float m_blk = fmaxf(mx0, mx1) * c;
      // move the reference maximum (and rescale O, l) only when P would exceed 2^8
      const bool move = m_blk > m + kRescaleAbove;
      const float m_new = move ? m_blk : m;
      const float alpha = move ? ex2_approx(m - m_new) : 1.f;  // 0 at j = 0 (m = -inf)
      const uint64_t c2 = f2pack(c, c), nm2 = f2pack(-m_new, -m_new);
      uint64_t sum2 = f2pack(0.f, 0.f);
      uint32_t pw[32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t(&a)[32] = cc ? a1 : a0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 z = f2unpack(
              ffma2(f2pack(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1])), c2, nm2));
          const float p0 = ex2_approx(z.x), p1 = ex2_approx(z.y);
          sum2 = fadd2(sum2, f2pack(p0, p1));
          pw[cc * 16 + e] = pack_bf16x2(p0, p1);
        }
      }
      const float2 sp = f2unpack(sum2);
      l = fmaf(l, alpha, sp.x + sp.y);
      m = m_new;
      // P V of the previous block has finished: its P buffer is free and O is stable
      if (j >= 1) {
        if (!wait_all(pv_full, (j - 1) & 1)) { ok = false; break; }
        tc_fence_after_sync();
      }
#pragma unroll
      for (int t = 0; t < 8; ++t)  // 16-byte chunk t of the row (8 keys), swizzled
        sts128(p_row + ((t ^ (r & 7)) << 4),
               make_uint4(pw[4 * t], pw[4 * t + 1], pw[4 * t + 2], pw[4 * t + 3]));
      if (j >= 1) {
        if (__any_sync(0xffffffffu, move)) {
          // O *= alpha for this warp's rows (alpha = 1 for rows that keep their reference)
          uint32_t o0[32], o1[32];
          tmem_ld32_async(t_lane + kTmemO, o0);
          tmem_ld32_async(t_lane + kTmemO + 32, o1);
          tmem_wait_ld();
          reg_fence(o0);
          reg_fence(o1);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            o0[e] = __float_as_uint(__uint_as_float(o0[e]) * alpha);
            o1[e] = __float_as_uint(__uint_as_float(o1[e]) * alpha);
          }
          tmem_st32(t_lane + kTmemO, o0);
          tmem_st32(t_lane + kTmemO + 32, o1);
          tmem_wait_st();
        }
      }
      // P_j is in shared memory and O rescaled: visible to the tensor cores, signalled
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = wait_all(pv_full, (nkb - 1) & 1);
    tc_fence_after_sync();
    const int row = q0 + r;
    if (ok) {
      uint32_t o0[32], o1[32];
      tmem_ld32_async(t_lane + kTmemO, o0);
      tmem_ld32_async(t_lane + kTmemO + 32, o1);
      tmem_wait_ld();
      reg_fence(o0);
      reg_fence(o1);
      if (row < p.L) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.L + row) * p.C +
                                              head * kHd);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          dst[v] = make_uint4(
              pack_bf16x2(__uint_as_float(o0[8 * v]) * inv, __uint_as_float(o0[8 * v + 1]) * inv),
              pack_bf16x2(__uint_as_float(o0[8 * v + 2]) * inv, __uint_as_float(o0[8 * v + 3]) * inv),
              pack_bf16x2(__uint_as_float(o0[8 * v + 4]) * inv, __uint_as_float(o0[8 * v + 5]) * inv),
              pack_bf16x2(__uint_as_float(o0[8 * v + 6]) * inv, __uint_as_float(o0[8 * v + 7]) * inv));
          dst[4 + v] = make_uint4(
              pack_bf16x2(__uint_as_float(o1[8 * v]) * inv, __uint_as_float(o1[8 * v + 1]) * inv),
              pack_bf16x2(__uint_as_float(o1[8 * v + 2]) * inv, __uint_as_float(o1[8 * v + 3]) * inv),
              pack_bf16x2(__uint_as_float(o1[8 * v + 4]) * inv, __uint_as_float(o1[8 * v + 5]) * inv),
              pack_bf16x2(__uint_as_float(o1[8 * v + 6]) * inv, __uint_as_float(o1[8 * v + 7]) * inv));
        }
      }
    }
    tc_fence_before_sync();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t attn_smem_bytes() { return static_cast<size_t>(smem_bytes()); }

int attn_q_box_rows() { return kQRows; }
int attn_kv_box_rows() { return kKeys; }

cudaError_t launch_attn(const CUtensorMap& tmQ, const CUtensorMap& tmKV, const AttnParams& p,
                        cudaStream_t stream, bool pdl) {
  const int smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.L + kQRows - 1) / kQRows, p.heads, p.B);
  return launch(attn_fwd_kernel, grid, dim3(kThreads), static_cast<size_t>(smem), stream, pdl,
                tmQ, tmKV, p);
}

}  // namespace rs
