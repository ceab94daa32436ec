// rs_fused.cu -- the whole MLP sublayer of "Representation Shift: Unifying Token
// Compression with FlashAttention" (§3.3 Eq. (6), with the shift of Eq. (4)) in
// one persistent tcgen05 kernel for narrow blocks (C <= 384), so that the
// hidden activation never leaves the SM.
//
// One CTA per SM takes 128-row tiles of x' round robin. Per tile:
//   for every 128-column chunk j of the hidden layer:
//     fc1   A1 = the x' tile (loaded once per tile by TMA, resident in shared
//           memory), B1 = Wg[128 j .. 128 j + 127, :] (LN-folded fc1 weights,
//           TMA ring) -> TMEM accumulator T1 (128 columns)
//     epilogue 1: z = rstd (T1 - mean G) + cb, a = bf16(GELU(z)), written to
//           shared memory in the UMMA operand layout (128-byte swizzle, K-major)
//     fc2   A2 = a, B2 = W2[:, 128 j .. 128 j + 127] (TMA ring, pieces of PR
//           output columns) -> TMEM accumulator T2 (C columns), summed over j
//   epilogue 2: h = T2 + b2, y = bf16(x' + h) through TMA-store boxes, and per
//     row and column quarter the partial sum of (h - x')^2 (four per row).
// TMEM: T2 in columns [0, C), T1 in [384, 512). The MMA warp issues fc1(j + 1)
// before fc2(j), so the tensor cores run the next chunk while the epilogue warps
// evaluate chunk j's GELU; T1 goes back to the MMA warp as soon as its values
// are in registers.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps
// 4..19 epilogue (lane quadrant q = warp % 4; column group = (warp - 4) / 4).
// Every wait is bounded (see rs_ptx.cuh): a wait that runs out records
// RS_ERR_DEVICE_TIMEOUT, all roles stop, in-flight MMAs and copies are drained
// and TMEM is freed before the CTA exits.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rs_internal.h"
#include "rs_ptx.cuh"
#include "rs_gelu.cuh"

namespace rs {
namespace {

constexpr int kFBM = 128;                   // rows of a tile
constexpr int kFBH = 128;                   // hidden columns per chunk (fc1 N, fc2 K)
constexpr int kFBK = 64;                    // one 128-byte swizzle row of bf16
constexpr int kFBlk = kFBM * kFBK * 2;      // 16 KB: one [128 x 64] operand block
constexpr int kFMaxKB1 = kFusedMaxC / kFBK; // fc1 k-blocks at most (C <= 384)
constexpr int kFStages = 4;                 // weight ring of 16 KB stages
constexpr int kFEpiWarp0 = 4;
constexpr int kFEpiWarps = 16;
constexpr int kFThreads = (kFEpiWarp0 + kFEpiWarps) * 32;
constexpr uint32_t kFT1Col = 384;           // T1 columns [384, 512)
constexpr int kFVecBytes = 2 * kFBH * 4;    // G and cb of one chunk (fp32)
constexpr int kFBoxCols = 16;                     // epilogue-2 output box: 32 x 16, 32-byte swizzle
constexpr int kFBoxBytes = kEpiBoxRows * kFBoxCols * 2;

// shared memory map, offsets from the 1024-byte aligned base
constexpr int kOffX = 0;                                   // x' tile: kFMaxKB1 blocks
constexpr int kOffH = kOffX + kFMaxKB1 * kFBlk;            // hidden chunk: 2 blocks
constexpr int kOffRing = kOffH + 2 * kFBlk;                // weight ring
constexpr int kOffBox = kOffRing + kFStages * kFBlk;       // epilogue-2 output boxes
constexpr int kOffVec = kOffBox + kFEpiWarps * kFBoxBytes; // G, cb: two chunks
constexpr int kOffB2 = kOffVec + 2 * kFVecBytes;           // b2 (bf16, C <= 384)
constexpr int kOffCtrl = kOffB2 + kFusedMaxC * 2;          // barriers, TMEM slot, abort flag
constexpr int kNumBars = 2 * kFStages + 13;
constexpr size_t kFSmem = 1024 + kOffCtrl + kNumBars * 8 + 16;

static_assert(kOffRing % 1024 == 0 && kOffH % 1024 == 0, "operand blocks 1024-byte aligned");
static_assert(kFSmem <= 232448, "shared memory");

template <int PR>
__global__ void __launch_bounds__(kFThreads, 1)
    mlp_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWg,
                     const __grid_constant__ CUtensorMap tmW2, const __grid_constant__ CUtensorMap tmY,
                     const FusedParams p) {
  static_assert(PR == 64 || PR == 128, "fc2 piece");
  constexpr uint32_t kIdesc1 = idesc_bf16_f32(kFBM, kFBH);
  constexpr uint32_t kIdesc2 = idesc_bf16_f32(kFBM, PR);
  constexpr uint32_t kW2Bytes = PR * kFBK * 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sX = smem + kOffX;
  uint8_t* sH = smem + kOffH;
  uint8_t* sRing = smem + kOffRing;
  uint8_t* sBox = smem + kOffBox;
  uint8_t* sVec = smem + kOffVec;
  uint8_t* sB2 = smem + kOffB2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffCtrl);
  uint64_t* full = bars;                    // [kFStages]
  uint64_t* empty = bars + kFStages;        // [kFStages]
  uint64_t* x_full = bars + 2 * kFStages;
  uint64_t* x_empty = x_full + 1;
  uint64_t* t1_full = x_full + 2;
  uint64_t* t1_empty = x_full + 3;
  uint64_t* h_full = x_full + 4;
  uint64_t* h_empty = x_full + 5;
  uint64_t* t2_full = x_full + 6;
  uint64_t* t2_empty = x_full + 7;
  uint64_t* vfull = x_full + 8;             // [2]
  uint64_t* vempty = x_full + 10;           // [2]
  uint64_t* drain = x_full + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int KB1 = p.C / kFBK;   // fc1 k-blocks
  const int NPC = p.C / PR;     // fc2 pieces per k-block
  const int J = p.H / kFBH;     // hidden chunks per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(x_full, 1);
    mbar_init(x_empty, 1);
    mbar_init(t1_full, 1);
    mbar_init(t1_empty, kFEpiWarps);
    mbar_init(h_full, kFEpiWarps);
    mbar_init(h_empty, 1);
    mbar_init(t2_full, 1);
    mbar_init(t2_empty, kFEpiWarps);
    for (int v = 0; v < 2; ++v) {
      mbar_init(&vfull[v], 1);
      mbar_init(&vempty[v], kFEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmWg);
    tma_prefetch_desc(&tmW2);
    tma_prefetch_desc(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < p.C / 8; i += blockDim.x)
    reinterpret_cast<uint4*>(sB2)[i] = __ldg(reinterpret_cast<const uint4*>(p.b2) + i);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Ring order = MMA order: Wg(0), then Wg(j), W2(j - 1) for j = 1 .. J-1, then
    // W2(J - 1); each chunk's G/cb slice ahead of its Wg blocks.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pend[kFStages];
#pragma unroll
      for (int s = 0; s < kFStages; ++s) pend[s] = -1;
      int xpend = -1, vpend0 = -1, vpend1 = -1;
      uint32_t xph = 0;
      int chunk = 0;  // chunks started by this CTA (G/cb buffer and phase)
      auto ring_load = [&](const CUtensorMap* map, int cx, int cy, uint32_t bytes) -> bool {
        if (!wait_bounded(&empty[stage], phase ^ 1u, wc)) return false;
        mbar_arrive_expect_tx(&full[stage], bytes);
        tma_load_2d(sRing + stage * kFBlk, map, &full[stage], cx, cy);
#pragma unroll
        for (int s = 0; s < kFStages; ++s)
          if (s == stage) pend[s] = static_cast<int>(phase);
        if (++stage == kFStages) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      auto vec_load = [&](int j) -> bool {
        const int vb = chunk & 1;
        const uint32_t vph = static_cast<uint32_t>(chunk >> 1) & 1u;
        if (!wait_bounded(&vempty[vb], vph ^ 1u, wc)) return false;
        mbar_arrive_expect_tx(&vfull[vb], kFVecBytes);
        uint8_t* dst = sVec + vb * kFVecBytes;
        bulk_load(dst, p.colG + j * kFBH, kFBH * 4, &vfull[vb]);
        bulk_load(dst + kFBH * 4, p.colC + j * kFBH, kFBH * 4, &vfull[vb]);
        if (vb == 0) vpend0 = static_cast<int>(vph); else vpend1 = static_cast<int>(vph);
        ++chunk;
        return true;
      };
      auto wg_chunk = [&](int j) -> bool {
        for (int kb = 0; kb < KB1; ++kb)
          if (!ring_load(&tmWg, kb * kFBK, j * kFBH, kFBlk)) return false;
        return true;
      };
      auto w2_chunk = [&](int j) -> bool {
        for (int kk = 0; kk < kFBH / kFBK; ++kk)
          for (int pc = 0; pc < NPC; ++pc)
            if (!ring_load(&tmW2, j * kFBH + kk * kFBK, pc * PR, kW2Bytes)) return false;
        return true;
      };
      bool ok = true;
      for (int mb = blockIdx.x; mb < p.num_m && ok; mb += gridDim.x) {
        if (!wait_bounded(x_empty, xph ^ 1u, wc)) break;
        mbar_arrive_expect_tx(x_full, static_cast<uint32_t>(KB1 * kFBlk));
        for (int kb = 0; kb < KB1; ++kb)
          tma_load_2d(sX + kb * kFBlk, &tmX, x_full, kb * kFBK, mb * kFBM);
        xpend = static_cast<int>(xph);
        xph ^= 1u;
        ok = vec_load(0) && wg_chunk(0);
        for (int j = 1; j < J && ok; ++j) ok = vec_load(j) && wg_chunk(j) && w2_chunk(j - 1);
        ok = ok && w2_chunk(J - 1);
      }
      // Every copy this thread issued must land before the CTA may exit.
#pragma unroll
      for (int s = 0; s < kFStages; ++s)
        if (pend[s] >= 0) wait_bounded(&full[s], static_cast<uint32_t>(pend[s]), wc, false);
      if (xpend >= 0) wait_bounded(x_full, static_cast<uint32_t>(xpend), wc, false);
      if (vpend0 >= 0) wait_bounded(&vfull[0], static_cast<uint32_t>(vpend0), wc, false);
      if (vpend1 >= 0) wait_bounded(&vfull[1], static_cast<uint32_t>(vpend1), wc, false);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t xph = 0, t1n = 0, hn = 0, t2n = 0;  // completed uses of each resource
      bool issued = false;
      auto ring_wait = [&]() -> bool {
        if (!wait_bounded(&full[stage], phase, wc)) return false;
        tc_fence_after_sync();
        return true;
      };
      auto ring_next = [&]() {
        umma_commit(&empty[stage]);
        if (++stage == kFStages) {
          stage = 0;
          phase ^= 1u;
        }
      };
      auto fc1 = [&](int j) -> bool {
        if (!wait_bounded(t1_empty, (t1n & 1u) ^ 1u, wc)) return false;
        tc_fence_after_sync();
        const uint32_t d = tmem_base + kFT1Col;
        for (int kb = 0; kb < KB1; ++kb) {
          if (!ring_wait()) return false;
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sX + kb * kFBlk));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sRing + stage * kFBlk));
#pragma unroll
          for (int k = 0; k < kFBK / 16; ++k)
            umma_bf16(d, ad + 2u * k, bd + 2u * k, kIdesc1, (kb | k) != 0 ? 1u : 0u);
          issued = true;
          ring_next();
        }
        umma_commit(t1_full);
        ++t1n;
        if (j == J - 1) umma_commit(x_empty);  // the tile's last read of x'
        return true;
      };
      auto fc2 = [&](int j) -> bool {
        if (!wait_bounded(h_full, hn & 1u, wc)) return false;
        if (j == 0 && !wait_bounded(t2_empty, (t2n & 1u) ^ 1u, wc)) return false;
        tc_fence_after_sync();
        for (int kk = 0; kk < kFBH / kFBK; ++kk) {
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sH + kk * kFBlk));
          for (int pc = 0; pc < NPC; ++pc) {
            if (!ring_wait()) return false;
            const uint64_t bd = sw128_kmajor_desc(smem_u32(sRing + stage * kFBlk));
            const uint32_t d = tmem_base + static_cast<uint32_t>(pc * PR);
#pragma unroll
            for (int k = 0; k < kFBK / 16; ++k)
              umma_bf16(d, ad + 2u * k, bd + 2u * k, kIdesc2, (j | kk | k) != 0 ? 1u : 0u);
            issued = true;
            ring_next();
          }
        }
        umma_commit(h_empty);  // the hidden chunk may be overwritten
        ++hn;
        if (j == J - 1) {
          umma_commit(t2_full);
          ++t2n;
        }
        return true;
      };
      bool ok = true;
      for (int mb = blockIdx.x; mb < p.num_m && ok; mb += gridDim.x) {
        if (!wait_bounded(x_full, xph, wc)) break;
        xph ^= 1u;
        tc_fence_after_sync();
        ok = fc1(0);
        for (int j = 1; j < J && ok; ++j) ok = fc1(j) && fc2(j - 1);
        ok = ok && fc2(J - 1);
      }
      if (*abort_flag && issued) {
        // Drain: wait until every MMA issued so far has finished with TMEM and smem.
        umma_commit(drain);
        wait_bounded(drain, 0u, wc, false);
      }
    }
    __syncwarp();
  } else if (warp >= kFEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quadrant: rows 32q .. 32q + 31
    const int grp = (warp - kFEpiWarp0) >> 2;  // column group 0..3
    const int r = q * 32 + lane;               // this lane's row in the tile
    uint8_t* box = sBox + (warp - kFEpiWarp0) * kFBoxBytes;
    const uint32_t box_u32 = smem_u32(box);
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const int cq = p.C / 4;  // epilogue-2 columns of this warp
    const int nch2 = cq / 16;
    uint32_t t1n = 0, hn = 0, t2n = 0;
    int chunk = 0;
    bool ok = true;
    for (int mb = blockIdx.x; mb < p.num_m && ok; mb += gridDim.x) {
      const int row = mb * kFBM + r;
      const bool row_ok = row < p.M;
      float2 st = make_float2(0.f, 0.f);
      if (row_ok) st = p.stats[row];
      const uint64_t nmu2 = f2pack(-st.x, -st.x);
      const uint64_t rs2 = f2pack(st.y, st.y);
      for (int j = 0; j < J; ++j) {
        // ---- epilogue 1: T1 -> fold + GELU -> bf16 hidden chunk in shared memory
        const int vb = chunk & 1;
        const uint32_t vph = static_cast<uint32_t>(chunk >> 1) & 1u;
        int w_ok = 1;
        if (lane == 0)
          w_ok = (wait_bounded(&vfull[vb], vph, wc) && wait_bounded(t1_full, t1n & 1u, wc)) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        mbar_try_wait(&vfull[vb], vph);  // completed: acquire for every lane
        mbar_try_wait(t1_full, t1n & 1u);
        tc_fence_after_sync();
        uint32_t ra[16], rb[16];
        tmem_ld16_async(tq + kFT1Col + grp * 32, ra);
        tmem_ld16_async(tq + kFT1Col + grp * 32 + 16, rb);
        tmem_wait_ld();
        reg_fence16(ra);
        reg_fence16(rb);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(t1_empty);
        ++t1n;
        const uint32_t vec_u32 = smem_u32(sVec + vb * kFVecBytes);
        uint32_t outw[16];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t(&rr)[16] = hh ? rb : ra;
          const uint32_t cvec = static_cast<uint32_t>(grp * 32 + hh * 16);
          uint64_t z2[8], g2[8];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 g4 = lds128(vec_u32 + (cvec + 4 * v) * 4);
            const uint4 c4 = lds128(vec_u32 + kFBH * 4 + (cvec + 4 * v) * 4);
            const uint64_t ga = (static_cast<uint64_t>(g4.y) << 32) | g4.x;
            const uint64_t gb = (static_cast<uint64_t>(g4.w) << 32) | g4.z;
            const uint64_t ca = (static_cast<uint64_t>(c4.y) << 32) | c4.x;
            const uint64_t cb = (static_cast<uint64_t>(c4.w) << 32) | c4.z;
            z2[2 * v] = ffma2(
                rs2,
                ffma2(nmu2, ga, f2pack(__uint_as_float(rr[4 * v]), __uint_as_float(rr[4 * v + 1]))),
                ca);
            z2[2 * v + 1] = ffma2(
                rs2,
                ffma2(nmu2, gb,
                      f2pack(__uint_as_float(rr[4 * v + 2]), __uint_as_float(rr[4 * v + 3]))),
                cb);
          }
          gelu2_block<8>(z2, g2);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 g = f2unpack(g2[e]);
            outw[hh * 8 + e] = pack_bf16x2(g.x, g.y);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&vempty[vb]);
        ++chunk;
        // the hidden buffer is free once fc2 of the previous chunk has read it
        if (lane == 0) w_ok = wait_bounded(h_empty, (hn & 1u) ^ 1u, wc) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) {
          ok = false;
          break;
        }
        mbar_try_wait(h_empty, (hn & 1u) ^ 1u);
        ++hn;
        {
          // columns 32 grp .. 32 grp + 31 of the chunk: operand block grp / 2,
          // 16-byte pieces 4 (grp % 2) .. +3 of row r, swizzled by r % 8
          const uint32_t hb = smem_u32(sH) + static_cast<uint32_t>((grp >> 1) * kFBlk + r * 128);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t c16 = static_cast<uint32_t>((grp & 1) * 4 + i);
            sts128(hb + ((c16 ^ static_cast<uint32_t>(r & 7)) << 4),
                   make_uint4(outw[4 * i], outw[4 * i + 1], outw[4 * i + 2], outw[4 * i + 3]));
          }
        }
        fence_proxy_async_smem();  // the MMA reads the chunk through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(h_full);
      }
      if (!ok) break;
      // ---- epilogue 2: T2 + b2, residual, y through TMA stores, shift partials
      {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_bounded(t2_full, t2n & 1u, wc) ? 1 : 0;
        w_ok = __shfl_sync(0xffffffffu, w_ok, 0);
        if (!w_ok) break;
        mbar_try_wait(t2_full, t2n & 1u);
        ++t2n;
        tc_fence_after_sync();
      }
      const int col0 = grp * cq;
      const uint32_t t_row = tq + static_cast<uint32_t>(col0);
      const uint32_t b2_u32 = smem_u32(sB2) + static_cast<uint32_t>(col0 * 2);
      const uint4* xrow = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(row) * p.C + col0);
      const bool box_live = mb * kFBM + q * 32 < p.M;
      float part = 0.f;
      uint32_t ra[16], rb[16];
      uint4 xa[2] = {}, xb[2] = {};
      tmem_ld16_async(t_row, ra);
      if (row_ok) {
        xa[0] = __ldg(xrow);
        xa[1] = __ldg(xrow + 1);
      }
      for (int n = 0; n < nch2; ++n) {
        uint32_t(&rr)[16] = (n & 1) ? rb : ra;
        uint32_t(&nx)[16] = (n & 1) ? ra : rb;
        uint4(&xv)[2] = (n & 1) ? xb : xa;
        uint4(&xn)[2] = (n & 1) ? xa : xb;
        tmem_wait_ld();
        reg_fence16(rr);
        if (n + 1 < nch2) {
          tmem_ld16_async(t_row + (n + 1) * 16, nx);
          if (row_ok) {
            xn[0] = __ldg(xrow + (n + 1) * 2);
            xn[1] = __ldg(xrow + (n + 1) * 2 + 1);
          }
        } else {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(t2_empty);
        }
        const uint4 b0 = lds128(b2_u32 + n * 32);
        const uint4 b1 = lds128(b2_u32 + n * 32 + 16);
        const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const uint32_t* xw = reinterpret_cast<const uint32_t*>(xv);
        uint32_t outw[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x0 = bf16lo(xw[e]), x1 = bf16hi(xw[e]);
          const float h0 = __uint_as_float(rr[2 * e]) + bf16lo(bw[e]);
          const float h1 = __uint_as_float(rr[2 * e + 1]) + bf16hi(bw[e]);
          outw[e] = pack_bf16x2(x0 + h0, x1 + h1);
          const float d0 = h0 - x0, d1 = h1 - x1;
          part = fmaf(d0, d0, part);
          part = fmaf(d1, d1, part);
        }
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
        const uint32_t sw = (lane >> 2) & 1;
        sts128(box_u32 + lane * 32 + ((0u ^ sw) << 4), make_uint4(outw[0], outw[1], outw[2], outw[3]));
        sts128(box_u32 + lane * 32 + ((1u ^ sw) << 4), make_uint4(outw[4], outw[5], outw[6], outw[7]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && box_live) {
          tma_store_2d(&tmY, box, col0 + n * 16, mb * kFBM + q * 32);
          bulk_commit_group();
        }
      }
      if (row_ok) p.partials[static_cast<size_t>(row) * kFusedPartials + grp] = part;
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int PR>
cudaError_t launch_fused_t(const CUtensorMap& tmX, const CUtensorMap& tmWg, const CUtensorMap& tmW2,
                           const CUtensorMap& tmY, const FusedParams& p, int num_sms,
                           cudaStream_t stream, bool pdl) {
  auto kern = mlp_fused_kernel<PR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFSmem));
  if (e != cudaSuccess) return e;
  const int grid = p.num_m < num_sms ? p.num_m : num_sms;
  return launch(kern, grid, kFThreads, kFSmem, stream, pdl, tmX, tmWg, tmW2, tmY, p);
}

}  // namespace

int fused_w2_rows(int C) { return C % 128 == 0 ? 128 : 64; }

cudaError_t launch_mlp_fused(const CUtensorMap& tmX, const CUtensorMap& tmWg,
                             const CUtensorMap& tmW2, const CUtensorMap& tmY, const FusedParams& p,
                             int num_sms, cudaStream_t stream, bool pdl) {
  if (!fused_supported(p.C, p.H)) return cudaErrorInvalidValue;
  if (fused_w2_rows(p.C) == 128)
    return launch_fused_t<128>(tmX, tmWg, tmW2, tmY, p, num_sms, stream, pdl);
  return launch_fused_t<64>(tmX, tmWg, tmW2, tmY, p, num_sms, stream, pdl);
}

}  // namespace rs
