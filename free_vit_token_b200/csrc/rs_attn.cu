// rs_attn.cu -- the attention core of the ViT attention sublayer on sm_100a:
// per sample and head, O = Softmax(Q K^T / sqrt(d)) V (Eq. (1) of
// "Representation Shift: Unifying Token Compression with FlashAttention", one
// head of width d = 64), without materialising the L x L score matrix.
//
// One CTA owns 128 queries of one (sample, head) and walks the keys in blocks
// of 64 (online softmax); two CTAs share an SM (256 TMEM columns and ~97 KB of
// shared memory each), so one CTA's softmax overlaps the other's loads and MMAs:
//   warp 0      TMA producer: the Q tile once, then K and V tiles of each key
//               block into a three-stage ring (3-D tensor maps over [B, L, 3C],
//               so rows past a sample's L read as zero and never cross samples);
//   warp 1      owns the CTA's TMEM columns and issues the MMAs:
//               S_j = Q K_j^T (M = 128, N = 64, K = 64) into one of two TMEM
//               score buffers, PV_j = P_j V_j (M = 128, N = 64, K = 64, V read
//               MN-major) into one of two TMEM output buffers;
//   warps 2..5  softmax, one query row per thread (its TMEM lane): row maximum
//               over the block, P = 2^(S log2(e)/sqrt(d) - m) rounded to bf16
//               into shared memory (the A operand of PV, 128-byte swizzle), the
//               running sum l, and O = alpha O + PV_{j-1} in registers; at the
//               end O / l goes out as bf16.
// The score buffers and P alternate, so S_{j+1} is computed and PV_j runs while
// the softmax of block j+1 proceeds. Every wait is bounded (timeout -> error
// flag, CTA abort, drain, TMEM freed).
#include <cstdint>

#include "rs_internal.h"
#include "rs_ptx.cuh"

namespace rs {

namespace {

constexpr int kHd = 64;                         // head width d
constexpr int kQRows = 128;                     // queries per CTA (TMEM lanes)
constexpr int kKeys = 64;                       // keys per block
constexpr int kKvStages = 3;
constexpr int kBox = kQRows * kHd * 2;          // the Q tile: 128 rows x 64 columns (16 KB)
constexpr int kKvBox = kKeys * kHd * 2;         // a K or V tile: 64 rows x 64 columns (8 KB)
constexpr int kPBytes = kQRows * kKeys * 2;     // P: 128 rows x 64 keys (16 KB)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemO = 2 * kKeys;          // PV buffers after the two score buffers
constexpr int kCtrl = 256;

constexpr int smem_bytes() {
  return 1024 + kBox + kKvStages * 2 * kKvBox + 2 * kPBytes + kCtrl;
}

__global__ void __launch_bounds__(kThreads, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmKV, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kBox;                       // stage s: K at sK + 2 kKvBox s, V after it
  uint8_t* sP = sK + kKvStages * 2 * kKvBox;     // buffer b at sP + kPBytes b
  uint64_t* q_full = reinterpret_cast<uint64_t*>(sP + 2 * kPBytes);
  uint64_t* k_full = q_full + 1;
  uint64_t* v_full = k_full + kKvStages;
  uint64_t* kv_empty = v_full + kKvStages;
  uint64_t* s_full = kv_empty + kKvStages;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_full = p_full + 2;
  uint64_t* drain = pv_full + 2;
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
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&pv_full[i], 1);
    }
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
      int issued = 0;
      for (int j = 0; j < nkb; ++j) {
        const int s = j % kKvStages;
        if (j >= kKvStages && !wait_bounded(&kv_empty[s], ((j / kKvStages) - 1) & 1, wc)) break;
        mbar_arrive_expect_tx(&k_full[s], kKvBox);
        tma_load_3d(sKs(s), &tmKV, &k_full[s], C + head * kHd, j * kKeys, b);
        mbar_arrive_expect_tx(&v_full[s], kKvBox);
        tma_load_3d(sVs(s), &tmKV, &v_full[s], 2 * C + head * kHd, j * kKeys, b);
        issued = j + 1;
      }
      // every load issued has landed before the CTA may finish (after an abort too)
      wait_bounded(q_full, 0u, wc, false);
      for (int j = issued > kKvStages ? issued - kKvStages : 0; j < issued; ++j) {
        wait_bounded(&k_full[j % kKvStages], (j / kKvStages) & 1, wc, false);
        wait_bounded(&v_full[j % kKvStages], (j / kKvStages) & 1, wc, false);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(kQRows, kKeys);
      constexpr uint32_t kIdO = idesc_bf16_f32_bmn(kQRows, kHd);
      const uint32_t q_u32 = smem_u32(sQ);
      auto issue_pv = [&](int i) -> bool {
        const int pb = i & 1, st = i % kKvStages;
        if (!wait_bounded(&p_full[pb], (i >> 1) & 1, wc)) return false;
        if (!wait_bounded(&v_full[st], (i / kKvStages) & 1, wc)) return false;
        tc_fence_after_sync();
        const uint32_t p_u32 = smem_u32(sP + pb * kPBytes);
        const uint32_t v_u32 = smem_u32(sVs(st));
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint64_t ad = sw128_kmajor_desc(p_u32) + kk * 2;
          const uint64_t bd = sw128_mnmajor_desc(v_u32 + kk * 2048, kKvBox);
          umma_bf16(tmem + kTmemO + pb * kHd, ad, bd, kIdO, kk > 0 ? 1u : 0u);
        }
        umma_commit(&pv_full[pb]);
        umma_commit(&kv_empty[st]);
        return true;
      };
      bool ok = wait_bounded(q_full, 0u, wc);
      for (int j = 0; ok && j < nkb; ++j) {
        const int sb = j & 1, st = j % kKvStages;
        if (!wait_bounded(&k_full[st], (j / kKvStages) & 1, wc) ||
            (j >= 2 && !wait_bounded(&s_empty[sb], ((j >> 1) - 1) & 1, wc))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t k_u32 = smem_u32(sKs(st));
#pragma unroll
        for (int kk = 0; kk < kHd / 16; ++kk)
          umma_bf16(tmem + sb * kKeys, sw128_kmajor_desc(q_u32) + kk * 2,
                    sw128_kmajor_desc(k_u32) + kk * 2, kIdS, kk > 0 ? 1u : 0u);
        umma_commit(&s_full[sb]);
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
    float m = -INFINITY;                        // running maximum, in log2 units
    float l = 0.f;                              // running sum of P
    float alpha_prev = 0.f;
    uint64_t o2[kHd / 2];                       // O, two columns per register pair
#pragma unroll
    for (int e = 0; e < kHd / 2; ++e) o2[e] = f2pack(0.f, 0.f);
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(bar, parity, wc) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (ok) mbar_try_wait(bar, parity);  // completed: acquire for every lane
      return ok != 0;
    };
    // O = a O + PV_i (PV_i relative to the running maximum after block i)
    auto fold = [&](int i, float a) -> bool {
      if (!wait_all(&pv_full[i & 1], (i >> 1) & 1)) return false;
      tc_fence_after_sync();
      uint32_t v0[32], v1[32];
      const uint32_t t = t_lane + kTmemO + (i & 1) * kHd;
      tmem_ld32_async(t, v0);
      tmem_ld32_async(t + 32, v1);
      tmem_wait_ld();
      reg_fence(v0);
      reg_fence(v1);
      const uint64_t a2 = f2pack(a, a);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        o2[e] = ffma2(o2[e], a2, f2pack(__uint_as_float(v0[2 * e]), __uint_as_float(v0[2 * e + 1])));
        o2[16 + e] =
            ffma2(o2[16 + e], a2, f2pack(__uint_as_float(v1[2 * e]), __uint_as_float(v1[2 * e + 1])));
      }
      return true;
    };
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      const int sb = j & 1;
      if (!wait_all(&s_full[sb], (j >> 1) & 1)) { ok = false; break; }
      tc_fence_after_sync();
      const uint32_t ts = t_lane + sb * kKeys;
      const int kvalid = p.L - j * kKeys;       // keys of this block inside the sample (>= 1)
      // the block's 64 scores of this row, keys past the sample's end set to -inf
      uint32_t a0[32], a1[32];
      tmem_ld32_async(ts, a0);
      tmem_ld32_async(ts + 32, a1);
      tmem_wait_ld();
      reg_fence(a0);
      reg_fence(a1);
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
      const float m_new = fmaxf(m, fmaxf(mx0, mx1) * c);
      const float alpha = ex2_approx(m - m_new);
      // P = 2^(s c - m_new), two lanes per step, into shared memory (row r,
      // 128-byte swizzle); 2^-inf = 0 for the masked keys
      const uint32_t p_u32 = smem_u32(sP + sb * kPBytes) + r * 128;
      const uint64_t c2 = f2pack(c, c), nm2 = f2pack(-m_new, -m_new);
      uint64_t sum2 = f2pack(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t(&a)[32] = cc ? a1 : a0;
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 z = f2unpack(
              ffma2(f2pack(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1])), c2, nm2));
          const float p0 = ex2_approx(z.x), p1 = ex2_approx(z.y);
          sum2 = fadd2(sum2, f2pack(p0, p1));
          pw[e] = pack_bf16x2(p0, p1);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int chunk = cc * 4 + t;          // 16-byte chunk of the row (8 keys)
          const uint32_t addr = p_u32 + ((chunk ^ (r & 7)) << 4);
          sts128(addr, make_uint4(pw[4 * t], pw[4 * t + 1], pw[4 * t + 2], pw[4 * t + 3]));
        }
      }
      const float2 sp = f2unpack(sum2);
      const float sum = sp.x + sp.y;
      // the score buffer is read: the MMA warp may overwrite it
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);
      l = fmaf(l, alpha, sum);
      m = m_new;
      // P_j is in shared memory: visible to the tensor cores, then signalled
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
      if (j >= 1 && !fold(j - 1, alpha_prev)) { ok = false; break; }
      alpha_prev = alpha;
    }
    if (ok) ok = fold(nkb - 1, alpha_prev);
    tc_fence_before_sync();
    const int row = q0 + r;
    if (ok && row < p.L) {
      const float inv = 1.f / l;
      uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(b) * p.L + row) * p.C +
                                            head * kHd);
      uint32_t w[kHd / 2];
#pragma unroll
      for (int e = 0; e < kHd / 2; ++e) {
        const float2 v = f2unpack(o2[e]);
        w[e] = pack_bf16x2(v.x * inv, v.y * inv);
      }
#pragma unroll
      for (int v = 0; v < kHd / 8; ++v)
        dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }
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
