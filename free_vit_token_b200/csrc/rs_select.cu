// rs_select.cu -- score finalisation, per-sample top-k selection and the row
// gather of the pruned token set ("Representation Shift: Unifying Token
// Compression with FlashAttention", §3.1 pruned set x-tilde, §3.2 Eq. (4) and
// "dropped the tokens having the lowest k scores").
//
// select: one CTA per sample. s_t = sqrt(sum_j P[t, j]) in fp32 (fixed order),
//   then a 4-pass MSB-first radix select over the fp32 score bits of the patch
//   tokens (non-negative floats order like their bit patterns) finds the k-th
//   largest key T and how many keys equal to T are taken; an ordered ballot
//   compaction then writes [0] ++ ascending(kept t): every key > T, and the
//   keys == T with the lowest indices first.
// gather: one warp per kept row, 16-byte vector loads and streaming stores.
#include <cstdint>
#include <cuda_runtime.h>

#include "rs_internal.h"

namespace rs {

// Exclusive prefix count of `flag` over the block in thread order; `total`
// receives the block-wide count. Every thread of the block must call it.
__device__ __forceinline__ uint32_t block_exclusive_count(bool flag, uint32_t* s_warp,
                                                          uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  const uint32_t mine = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) s_warp[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < nw ? s_warp[lane] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    s_warp[lane] = incl - v;
    if (lane == 31) s_warp[32] = incl;
  }
  __syncthreads();
  const uint32_t res = s_warp[warp] + mine;
  total = s_warp[32];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ partials, int NP,
                                                      int L, int k, float* __restrict__ scores,
                                                      int32_t* __restrict__ kept) {
  extern __shared__ uint32_t s_key[];  // [L] fp32 score bits
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_warp[33];
  __shared__ uint32_t s_sel[2];
  const int b = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5;

  const float* P = partials + static_cast<size_t>(b) * L * NP;
  for (int t = tid; t < L; t += nt) {
    const float* pr = P + static_cast<size_t>(t) * NP;
    float acc = 0.f;
    for (int j = 0; j < NP; ++j) acc += pr[j];
    const float s = sqrtf(acc);
    scores[static_cast<size_t>(b) * L + t] = s;
    s_key[t] = __float_as_uint(s);
  }
  int32_t* out = kept + static_cast<size_t>(b) * (k + 1);
  if (tid == 0) out[0] = 0;  // CLS: always kept, never ranked
  if (k == 0) return;
  __syncthreads();

  // Radix select of the k-th largest key among t = 1..L-1.
  uint32_t prefix = 0, mask = 0, need = static_cast<uint32_t>(k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nt) s_hist[i] = 0;
    __syncthreads();
    for (int base = 1; base < L; base += nt) {
      const int t = base + tid;
      const uint32_t u = t < L ? s_key[t] : 0u;
      const bool cand = t < L && (u & mask) == prefix;
      const uint32_t digit = cand ? ((u >> shift) & 0xFFu) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, digit);
      if (cand && lane == __ffs(peers) - 1) atomicAdd(&s_hist[digit], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l (lane 0 the highest)
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = s_hist[255 - 8 * lane - i];
        sum += c[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      uint32_t above = incl - sum;
      if (above < need && need <= incl) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + c[i] >= need) {
            s_sel[0] = static_cast<uint32_t>(255 - 8 * lane - i);
            s_sel[1] = above;
            break;
          }
          above += c[i];
        }
      }
    }
    __syncthreads();
    prefix |= s_sel[0] << shift;
    mask |= 0xFFu << shift;
    need -= s_sel[1];
    __syncthreads();
  }
  const uint32_t T = prefix;  // k-th largest key; `need` keys equal to T are kept

  // Ordered compaction: ascending t.
  uint32_t eq_base = 0, out_base = 0;
  for (int base = 1; base < L; base += nt) {
    const int t = base + tid;
    const bool valid = t < L;
    const uint32_t u = valid ? s_key[t] : 0u;
    const bool gt = valid && u > T;
    const bool eq = valid && u == T;
    uint32_t eq_tot, keep_tot;
    const uint32_t eq_rank = eq_base + block_exclusive_count(eq, s_warp, eq_tot);
    const bool keep = gt || (eq && eq_rank < need);
    const uint32_t pos = out_base + block_exclusive_count(keep, s_warp, keep_tot);
    if (keep) out[1 + pos] = t;
    eq_base += eq_tot;
    out_base += keep_tot;
  }
}

template <int VPL>
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ y, int L, int Cv,
                                                     const int32_t* __restrict__ kept, int k1,
                                                     int rows_total, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  for (int row = gw; row < rows_total; row += nw) {
    const int b = row / k1;
    const int t = __ldg(kept + row);
    uint4* dst = out + static_cast<size_t>(row) * Cv;
    uint4 v[VPL];
    if (t >= 0 && t < L) {
      const uint4* src = y + (static_cast<size_t>(b) * L + t) * Cv;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const int idx = lane + 32 * i;
        if (idx < Cv) v[i] = __ldg(src + idx);
      }
    } else {
#pragma unroll
      for (int i = 0; i < VPL; ++i) v[i] = make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int idx = lane + 32 * i;
      if (idx < Cv) __stcs(dst + idx, v[i]);
    }
  }
}

cudaError_t launch_select(const float* partials, int num_partials, int B, int L, int keep_k,
                          float* scores, int32_t* kept_idx, cudaStream_t stream) {
  static bool attr_set = false;
  const size_t smem = static_cast<size_t>(L) * sizeof(uint32_t);
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         RS_MAX_L * static_cast<int>(sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int threads = ((L + 31) / 32) * 32;
  if (threads > 1024) threads = 1024;
  if (threads < 64) threads = 64;
  select_kernel<<<B, threads, smem, stream>>>(partials, num_partials, L, keep_k, scores, kept_idx);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* y, int B, int L, int C, const int32_t* kept_idx, int keep_k,
                          void* y_kept, int num_sms, cudaStream_t stream) {
  const int Cv = C / 8;
  const int k1 = keep_k + 1;
  const int rows = B * k1;
  int blocks = (rows + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  const auto* yp = static_cast<const uint4*>(y);
  auto* op = static_cast<uint4*>(y_kept);
  const int vpl = (Cv + 31) / 32;
  if (vpl <= 1)
    gather_kernel<1><<<blocks, 256, 0, stream>>>(yp, L, Cv, kept_idx, k1, rows, op);
  else if (vpl <= 2)
    gather_kernel<2><<<blocks, 256, 0, stream>>>(yp, L, Cv, kept_idx, k1, rows, op);
  else if (vpl <= 4)
    gather_kernel<4><<<blocks, 256, 0, stream>>>(yp, L, Cv, kept_idx, k1, rows, op);
  else
    gather_kernel<8><<<blocks, 256, 0, stream>>>(yp, L, Cv, kept_idx, k1, rows, op);
  return cudaGetLastError();
}

}  // namespace rs
