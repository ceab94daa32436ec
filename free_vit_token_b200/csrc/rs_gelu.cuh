// rs_gelu.cuh -- the exact (erf) GELU of the MLP (§3.3 Eq. (6) of "Representation
// Shift: Unifying Token Compression with FlashAttention"; GELU(z) = z * Phi(z)) on
// pairs of fp32 lanes, shared by the GEMM epilogue (rs_mlp.cu) and the fused MLP
// kernel (rs_fused.cu). Phi comes from the polynomials of rs_gelu_poly.h (fitted by
// gen_gelu_poly.py to the normal CDF).
#pragma once

#include <cstdint>

#include "rs_gelu_poly.h"
#include "rs_ptx.cuh"

namespace rs {

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t kpair(float c) { return f2pack(c, c); }

// Exact (erf) GELU of two fp32 lanes, GELU(z) = z * Phi(z), evaluated with the
// polynomial of rs_gelu_poly.h (max |error| 1.1e-6, max |Phi error| 2.5e-7 in
// float32) using paired fp32 FMAs:
//   u = min(K z^2 - 1, 1), Phi = sat(1/2 + z P(u)).
__device__ __forceinline__ uint64_t gelu2(uint64_t z2) {
  uint64_t u2 = ffma2(fmul2(z2, kpair(RS_GELU_K)), z2, kpair(-1.f));
  const float2 uf = f2unpack(u2);
  u2 = f2pack(fminf(uf.x, 1.f), fminf(uf.y, 1.f));
  uint64_t p = kpair(RS_GELU_P13);
  p = ffma2(p, u2, kpair(RS_GELU_P12));
  p = ffma2(p, u2, kpair(RS_GELU_P11));
  p = ffma2(p, u2, kpair(RS_GELU_P10));
  p = ffma2(p, u2, kpair(RS_GELU_P9));
  p = ffma2(p, u2, kpair(RS_GELU_P8));
  p = ffma2(p, u2, kpair(RS_GELU_P7));
  p = ffma2(p, u2, kpair(RS_GELU_P6));
  p = ffma2(p, u2, kpair(RS_GELU_P5));
  p = ffma2(p, u2, kpair(RS_GELU_P4));
  p = ffma2(p, u2, kpair(RS_GELU_P3));
  p = ffma2(p, u2, kpair(RS_GELU_P2));
  p = ffma2(p, u2, kpair(RS_GELU_P1));
  p = ffma2(p, u2, kpair(RS_GELU_P0));
  const float2 zf = f2unpack(z2), pf = f2unpack(p);
  return fmul2(z2, f2pack(__saturatef(fmaf(zf.x, pf.x, 0.5f)), __saturatef(fmaf(zf.y, pf.y, 0.5f))));
}

// Near-range GELU of two lanes, valid for |z| <= RS_GELU_NEAR_Z, given
// u = RS_GELU_NEAR_K z^2 - 1 (in [-1, 1] there): Phi = 1/2 + z P(u), degree 6,
// no clamp and no saturation (max |error| 1.5e-5, below a seventh of the bf16
// half-spacing of every output of magnitude >= 0.05 that the value is stored as).
__device__ __forceinline__ uint64_t gelu2_near(uint64_t z2, uint64_t u2) {
  uint64_t p = kpair(RS_GELU_NEAR_P6);
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P5));
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P4));
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P3));
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P2));
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P1));
  p = ffma2(p, u2, kpair(RS_GELU_NEAR_P0));
  return fmul2(z2, ffma2(z2, p, kpair(0.5f)));
}

// GELU of N lane pairs held by a warp: the near-range polynomial when every
// value the warp holds has |z| <= RS_GELU_NEAR_Z (a warp-uniform choice), the
// full-range one otherwise. Every lane of the warp must call it.
template <int N>
__device__ __forceinline__ void gelu2_block(const uint64_t (&z2)[N], uint64_t (&g2)[N]) {
  uint64_t u2[N];
  float um = -1.f;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    u2[i] = ffma2(fmul2(z2[i], kpair(RS_GELU_NEAR_K)), z2[i], kpair(-1.f));
    const float2 uf = f2unpack(u2[i]);
    um = fmaxf(um, fmaxf(uf.x, uf.y));
  }
  if (__all_sync(0xffffffffu, um <= 1.f)) {
#pragma unroll
    for (int i = 0; i < N; ++i) g2[i] = gelu2_near(z2[i], u2[i]);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) g2[i] = gelu2(z2[i]);
  }
}

}  // namespace rs
