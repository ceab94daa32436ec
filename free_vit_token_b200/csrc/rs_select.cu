// rs_select.cu -- score finalisation, per-sample top-k selection and the row
// gather of the pruned token set ("Representation Shift: Unifying Token
// Compression with FlashAttention", §3.1 pruned set x-tilde, §3.2 Eq. (4) and
// "dropped the tokens having the lowest k scores").
//
// Scores in fp32, partials added left to right (§3.3 "Distance metrics"):
// L2 s_t = sqrt(sum_j P[t, j]); L1 s_t = sum_j P[t, j]; cosine, from per-group
// triples (h.x, h.h, x.x): s_t = max(0, 1 - HX / max(sqrt(HH) sqrt(XX), 1e-8)).
// Selection compares fp32 score bits (non-negative floats order like their bit
// patterns). Token u beats token t when key_u > key_t, or key_u == key_t and
// u < t; the kept set is the k ranked tokens beaten by fewer than k others. With a
// CLS token the ranked tokens are t = 1..L-1 and the list is [0] ++ ascending(kept
// t) -- CLS first, never ranked; without, all L tokens are ranked.
//   * L <= 256: every thread holds one key and counts its beaters in one sweep
//     over shared memory; an ordered ballot compaction follows.
//   * longer L: an MSB-first radix select finds the k-th largest key T and how
//     many keys equal to T are kept; the ordered compaction keeps every key > T
//     and the lowest-index keys == T. It ranks key - kmin (kmin the smallest ranked
//     key), whose digits start at the highest set bit of kmax - kmin, so the first
//     digit already spreads the keys over the bins, and it stops refining as soon
//     as the bin holding the k-th key has at most 32 keys: one warp ranks those.
// Kernels: select (one CTA per sample), gather (warps share out each sample's
// kept rows), and select+gather fused (B x S CTAs: each CTA selects its
// sample's rows and copies every S-th kept row, so the copy spreads over the GPU).
#include <cstdint>
#include <cuda_runtime.h>

#include "rs_internal.h"
#include "rs_ptx.cuh"

namespace rs {

constexpr int kRankMaxL = 256;

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

// Exclusive prefix sum of `v` over the block in thread order; `total` receives
// the block-wide sum. Every thread of the block must call it.
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t v, uint32_t* s_warp,
                                                        uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < nw ? s_warp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    s_warp[lane] = wi - w;
    if (lane == 31) s_warp[32] = wi;
  }
  __syncthreads();
  const uint32_t res = s_warp[warp] + incl - v;
  total = s_warp[32];
  __syncthreads();
  return res;
}

// Number of ranked tokens u that beat key `key` of token t: key_u >= key for
// u < t, key_u > key for u > t (u = t never counts). The sweep is split at t so
// every key costs one compare. s_key holds L keys padded with zeros to a multiple
// of 4: a zero pad lies above t and is never > key. With a CLS token (cls), the
// CLS slot (u = 0 < t, counted exactly when key_0 >= key) is removed.
__device__ __forceinline__ uint32_t count_beaters(const uint32_t* s_key, int L, uint32_t key,
                                                  int t, bool cls) {
  const uint4* k4 = reinterpret_cast<const uint4*>(s_key);
  const int q = (L + 3) >> 2;
  const int qt = t >> 2;  // the quad holding t
  uint32_t n = 0;
#pragma unroll 4
  for (int i = 0; i < qt; ++i) {
    const uint4 v = k4[i];
    n += (v.x >= key) + (v.y >= key) + (v.z >= key) + (v.w >= key);
  }
  {
    const uint4 v = k4[qt];
    const int r = t & 3;
    n += r > 0 ? static_cast<uint32_t>(v.x >= key) : 0u;
    n += r > 1 ? static_cast<uint32_t>(v.y >= key) : (r < 1 ? static_cast<uint32_t>(v.y > key) : 0u);
    n += r > 2 ? static_cast<uint32_t>(v.z >= key) : (r < 2 ? static_cast<uint32_t>(v.z > key) : 0u);
    n += r < 3 ? static_cast<uint32_t>(v.w > key) : 0u;
  }
#pragma unroll 4
  for (int i = qt + 1; i < q; ++i) {
    const uint4 v = k4[i];
    n += (v.x > key) + (v.y > key) + (v.z > key) + (v.w > key);
  }
  return cls ? n - (s_key[0] >= key) : n;  // CLS is never ranked
}

// Shared memory of one selecting CTA.
struct SelSmem {
  uint32_t* key;   // [roundup(L, 4)] score bits, zero padded
  int32_t* kept;   // [k + 1] kept token list
  uint32_t* warp;  // [64] block scan scratch
  uint32_t* hist;  // [3][256] radix histograms (pass p uses p % 3), zero on entry to a pass
  uint32_t* sel;   // [8]: [0] T and [1] need from the candidate ranking; [6] counts
                   // the keys listed in cand (zero on entry to the selection)
  uint32_t* rng;   // [2]: the smallest and the largest ranked key of the sample
  uint32_t* cand;  // [2 * 32]: the final bin's keys [0, 32) and their tokens [32, 64)
};

__device__ __forceinline__ SelSmem carve(uint8_t* dyn, int L, uint32_t* s_warp, uint32_t* s_hist,
                                         uint32_t* s_sel, uint32_t* s_rng, uint32_t* s_cand) {
  SelSmem s;
  s.key = reinterpret_cast<uint32_t*>(dyn);
  s.kept = reinterpret_cast<int32_t*>(dyn + ((L + 3) & ~3) * 4);
  s.warp = s_warp;
  s.hist = s_hist;
  s.sel = s_sel;
  s.rng = s_rng;
  s.cand = s_cand;
  return s;
}

// Scores of sample b from its partials into s.key (and to `scores` when given).
// Each thread takes rows t = base + tid + i * nt (i < 4) per round and issues all
// of their loads before adding; the fp32 additions of a row run left to right.
__device__ __forceinline__ void load_keys(const float* __restrict__ partials, int NP, int L, int b,
                                          float* __restrict__ scores, const SelSmem& s, int dist,
                                          int first) {
  const int Lpad = (L + 3) & ~3;
  const int tid = threadIdx.x, nt = blockDim.x;
  const float* P = partials + static_cast<size_t>(b) * L * NP;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;  // over this thread's ranked keys (t >= first)
  auto store = [&](int t, float v) {
    if (scores != nullptr) scores[static_cast<size_t>(b) * L + t] = v;
    const uint32_t key = __float_as_uint(v);
    s.key[t] = key;
    if (t >= first) {
      kmin = key < kmin ? key : kmin;
      kmax = key > kmax ? key : kmax;
    }
  };
  // L2: sqrt of the summed squares; L1: the sum itself
  auto finish = [&](int t, float acc) { store(t, dist == kDistL2 ? sqrtf(acc) : acc); };
  if (dist == kDistCos) {
    // per-group triples (h.x, h.h, x.x), each component summed left to right
    for (int t = tid; t < Lpad; t += nt) {
      if (t < L) {
        const float* pr = P + static_cast<size_t>(t) * NP;
        float hx = 0.f, hh = 0.f, xx = 0.f;
        for (int j = 0; j < NP; j += 3) {
          hx += __ldg(pr + j);
          hh += __ldg(pr + j + 1);
          xx += __ldg(pr + j + 2);
        }
        const float den = fmaxf(sqrtf(hh) * sqrtf(xx), 1e-8f);
        store(t, fmaxf(1.0f - hx / den, 0.f));
      } else {
        s.key[t] = 0u;
      }
    }
  } else if ((NP & 3) == 0 && NP <= 8) {
    // NP a multiple of 4: every row 16-byte aligned, one or two quad loads per row
    const int np4 = NP >> 2;
    const float4* P4 = reinterpret_cast<const float4*>(P);
    for (int base = 0; base < Lpad; base += 4 * nt) {
      float4 v[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = base + tid + i * nt;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          v[i][j] = (t < L && j < np4) ? __ldg(P4 + static_cast<size_t>(t) * np4 + j)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = base + tid + i * nt;
        if (t < L) {
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j < np4) {
              acc += v[i][j].x;
              acc += v[i][j].y;
              acc += v[i][j].z;
              acc += v[i][j].w;
            }
          }
          finish(t, acc);
        } else if (t < Lpad) {
          s.key[t] = 0u;
        }
      }
    }
  } else if ((NP & 1) == 0 && NP <= 8) {
    // an even NP keeps every row 8-byte aligned: up to four pairs per row
    const int np2 = NP >> 1;
    const float2* P2 = reinterpret_cast<const float2*>(P);
    for (int base = 0; base < Lpad; base += 4 * nt) {
      float2 v[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = base + tid + i * nt;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          v[i][j] = (t < L && j < np2) ? __ldg(P2 + static_cast<size_t>(t) * np2 + j)
                                       : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = base + tid + i * nt;
        if (t < L) {
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j < np2) {
              acc += v[i][j].x;
              acc += v[i][j].y;
            }
          }
          finish(t, acc);
        } else if (t < Lpad) {
          s.key[t] = 0u;
        }
      }
    }
  } else {
    for (int t = tid; t < Lpad; t += nt) {
      if (t < L) {
        const float* pr = P + static_cast<size_t>(t) * NP;
        float acc = 0.f;
        for (int j = 0; j < NP; ++j) acc += __ldg(pr + j);
        finish(t, acc);
      } else {
        s.key[t] = 0u;
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if ((threadIdx.x & 31) == 0) {
    atomicMin(&s.rng[0], kmin);
    atomicMax(&s.rng[1], kmax);
  }
  __syncthreads();
}

// The selection's shared state before its first use: range bounds, histograms,
// candidate count and slots. Every thread calls it, before the kernel's
// dependency wait (so it overlaps the previous kernel's tail); it ends with a
// barrier.
__device__ __forceinline__ void init_select_smem(uint32_t* s_hist, uint32_t* s_sel, uint32_t* s_rng,
                                                 uint32_t* s_cand) {
  for (int i = threadIdx.x; i < 768; i += blockDim.x) s_hist[i] = 0;
  if (threadIdx.x < 64) s_cand[threadIdx.x] = 0u;
  if (threadIdx.x == 0) {
    s_sel[6] = 0;
    s_rng[0] = 0xFFFFFFFFu;
    s_rng[1] = 0u;
  }
  __syncthreads();
}

// The kept list of one sample into s.kept. Every thread of the block calls it;
// it ends with a barrier, so s.kept is complete on return.
__device__ void select_into_smem(int L, int k, const SelSmem& s, bool cls) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int first = cls ? 1 : 0;  // first ranked token; also the kept list's offset
  if (tid == 0 && cls) s.kept[0] = 0;
  if (k == 0) {
    __syncthreads();
    return;
  }
  if (L <= kRankMaxL && nt >= L) {
    const int t = tid;
    const uint32_t key = t < L ? s.key[t] : 0u;
    const bool keep =
        t >= first && t < L && count_beaters(s.key, L, key, t, cls) < static_cast<uint32_t>(k);
    uint32_t total;
    const uint32_t pos = block_exclusive_count(keep, s.warp, total);
    if (keep) s.kept[first + pos] = t;
    __syncthreads();
    return;
  }
  // Radix select of the k-th largest key among t = first..L-1. Each round of a pass
  // gives thread tid the four keys t = base + 4 tid .. +3 (one 16-byte load).
  const int Lpad = (L + 3) & ~3;
  const uint4* key4 = reinterpret_cast<const uint4*>(s.key);
  // Every ranked key lies in [kmin, kmax] (as unsigned integers). The select runs on
  // v = key - kmin in [0, kmax - kmin], which orders like the keys; its first digit
  // takes the 8 bits below the highest set bit of kmax - kmin, so it spreads the keys
  // over at least 128 bins however the range sits against powers of two (the fp32
  // exponent field).
  const int nw = nt >> 5;
  const uint32_t kmin = s.rng[0], kmax = s.rng[1];
  uint32_t T, need = static_cast<uint32_t>(k);  // keys == T kept, lowest index first
  if (kmin == kmax) {
    T = kmin;  // every ranked key is the same
  } else {
    int hb = 31 - __clz(kmax - kmin);  // highest bit of any v
    uint32_t mask = hb == 31 ? 0u : ~0u << (hb + 1);
    uint32_t prefix = 0;  // every v is zero above hb
    // Each pass: a histogram of the candidates' digit (bits hb .. shift of v, at most
    // 8) into buffer p % 3, one barrier, then every warp scans it for the bin holding
    // the need-th key. Buffer p % 3 is next written in pass p + 3 and zeroed during
    // pass p + 2, after every warp has passed the barrier of pass p + 1 and with it
    // its own scan of pass p.
    for (int pass = 0;; ++pass) {
      const int shift = hb >= 7 ? hb - 7 : 0;
      const uint32_t dmask = (2u << (hb - shift)) - 1u;
      uint32_t* hist = s.hist + 256 * (pass % 3);
      if (pass >= 2) {
        uint32_t* next = s.hist + 256 * ((pass + 1) % 3);
        for (int i = tid; i < 256; i += nt) next[i] = 0;
      }
      for (int base = 0; base < L; base += 4 * nt) {
        const int t0 = base + 4 * tid;
        const uint4 q = t0 < Lpad ? key4[t0 >> 2] : make_uint4(0, 0, 0, 0);
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = t0 + i;
          const uint32_t v = u[i] - kmin;
          if (t >= first && t < L && (v & mask) == prefix) atomicAdd(&hist[(v >> shift) & dmask], 1u);
        }
      }
      __syncthreads();
      // lane l owns digits 255-8l .. 248-8l (lane 0 the highest), two 16-byte loads
      const uint4* h4 = reinterpret_cast<const uint4*>(hist) + (62 - 2 * lane);
      const uint4 qlo = h4[0], qhi = h4[1];
      const uint32_t c[8] = {qhi.w, qhi.z, qhi.y, qhi.x, qlo.w, qlo.z, qlo.y, qlo.x};
      uint32_t sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) sum += c[i];
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      uint32_t above = incl - sum, digit = 0, in_bin = 0;
      const bool here = above < need && need <= incl;
      if (here) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + c[i] >= need) {
            digit = static_cast<uint32_t>(255 - 8 * lane - i);
            in_bin = c[i];
            break;
          }
          above += c[i];
        }
      }
      const int src = __ffs(__ballot_sync(0xffffffffu, here)) - 1;
      digit = __shfl_sync(0xffffffffu, digit, src);
      in_bin = __shfl_sync(0xffffffffu, in_bin, src);
      need -= __shfl_sync(0xffffffffu, above, src);  // now 1 <= need <= in_bin
      prefix |= digit << shift;
      mask |= dmask << shift;
      if (shift == 0) {
        T = prefix + kmin;  // the whole key is known
        break;
      }
      if (in_bin <= 32) {
        // The bin's keys into s.cand in any order (one shared atomic per warp round
        // that holds any of them), one barrier; every lane of warp 0 ranks one of them
        // against all (key descending, token ascending): the need-th is the k-th
        // ranked key overall, T its key, and the keys == T that are kept are `need`
        // minus the bin's keys above T; one barrier.
        for (int base = 0; base < L; base += 4 * nt) {
          const int t0 = base + 4 * tid;
          const uint4 q = t0 < Lpad ? key4[t0 >> 2] : make_uint4(0, 0, 0, 0);
          const uint32_t u[4] = {q.x, q.y, q.z, q.w};
          uint32_t bal[4], total = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int t = t0 + i;
            bal[i] = __ballot_sync(0xffffffffu,
                                   t >= first && t < L && ((u[i] - kmin) & mask) == prefix);
            total += __popc(bal[i]);
          }
          if (total != 0u) {
            uint32_t slot = 0;
            if (lane == 0) slot = atomicAdd(&s.sel[6], total);
            slot = __shfl_sync(0xffffffffu, slot, 0);
            const uint32_t below = (1u << lane) - 1u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if ((bal[i] >> lane) & 1u) {
                const uint32_t at = slot + __popc(bal[i] & below);
                s.cand[at] = u[i];
                s.cand[32 + at] = static_cast<uint32_t>(t0 + i);
              }
              slot += __popc(bal[i]);
            }
          }
        }
        __syncthreads();
        if (warp == 0) {
          // lane l holds candidate l as one 64-bit key, larger = ranked first (key
          // descending, token ascending; tokens differ, so no two are equal); the others
          // come by shuffle, one per step
          const bool mine = static_cast<uint32_t>(lane) < in_bin;
          const uint64_t kk = mine ? (static_cast<uint64_t>(s.cand[lane]) << 32) |
                                         static_cast<uint64_t>(~s.cand[32 + lane])
                                   : 0ull;
          uint32_t rank = 0;
#pragma unroll
          for (int j = 0; j < 32; ++j) rank += __shfl_sync(0xffffffffu, kk, j) > kk ? 1u : 0u;
          // invalid lanes hold 0, below every candidate: they never count against one
          const int at = __ffs(__ballot_sync(0xffffffffu, mine && rank == need - 1)) - 1;
          const uint32_t tkey = static_cast<uint32_t>(__shfl_sync(0xffffffffu, kk, at) >> 32);
          const uint32_t gt = __popc(__ballot_sync(0xffffffffu, mine && static_cast<uint32_t>(kk >> 32) > tkey));
          if (lane == 0) {
            s.sel[0] = tkey;
            s.sel[1] = need - gt;
          }
        }
        __syncthreads();
        T = s.sel[0];
        need = s.sel[1];
        break;
      }
      hb = shift - 1;
    }
  }
  // Ordered compaction: token t (first <= t < L) is kept when key_t > T, or key_t == T
  // and fewer than `need` equal keys precede it; its place among the kept tokens
  // is (#keys > T before t) + min(#keys == T before t, need). One packed count per
  // round (> T in the low half, == T in the high half): a warp scan, one barrier
  // for the warp totals (double-buffered across rounds), each warp's own offset.
  uint32_t gt_base = 0, eq_base = 0;
  for (int base = 0, round = 0; base < L; base += 4 * nt, ++round) {
    const int t0 = base + 4 * tid;
    const uint4 q = t0 < Lpad ? key4[t0 >> 2] : make_uint4(0, 0, 0, 0);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
    uint32_t gt_m = 0, eq_m = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + i;
      if (t >= first && t < L) {
        gt_m |= static_cast<uint32_t>(u[i] > T) << i;
        eq_m |= static_cast<uint32_t>(u[i] == T) << i;
      }
    }
    const uint32_t cnt = static_cast<uint32_t>(__popc(gt_m)) | (static_cast<uint32_t>(__popc(eq_m)) << 16);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    uint32_t* wb = s.warp + 32 * (round & 1);
    if (lane == 31) wb[warp] = incl;
    __syncthreads();
    const uint32_t wt = lane < nw ? wb[lane] : 0u;
    const uint32_t pre = __reduce_add_sync(0xffffffffu, lane < warp ? wt : 0u) + incl - cnt;
    const uint32_t tot = __reduce_add_sync(0xffffffffu, wt);
    uint32_t gtb = gt_base + (pre & 0xFFFFu), eqb = eq_base + (pre >> 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t gt = (gt_m >> i) & 1u, eq = (eq_m >> i) & 1u;
      if (gt || (eq && eqb < need)) s.kept[first + gtb + (eqb < need ? eqb : need)] = t0 + i;
      gtb += gt;
      eqb += eq;
    }
    gt_base += tot & 0xFFFFu;
    eq_base += tot >> 16;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ partials, int NP,
                                                      int L, int k, int dist, bool cls,
                                                      float* __restrict__ scores,
                                                      int32_t* __restrict__ kept) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ uint32_t s_warp[64], s_sel[8], s_rng[2];
  __shared__ __align__(16) uint32_t s_hist[768], s_cand[64];
  pdl_trigger();
  init_select_smem(s_hist, s_sel, s_rng, s_cand);
  pdl_wait();
  const int b = blockIdx.x;
  const SelSmem s = carve(dyn, L, s_warp, s_hist, s_sel, s_rng, s_cand);
  load_keys(partials, NP, L, b, scores, s, dist, cls ? 1 : 0);
  select_into_smem(L, k, s, cls);
  const int k1 = k + (cls ? 1 : 0);
  int32_t* out = kept + static_cast<size_t>(b) * k1;
  for (int i = threadIdx.x; i < k1; i += blockDim.x) out[i] = s.kept[i];
}

// Copies kept rows r = r_first, r_first + r_step, ... (r < k1) of sample b; a warp
// moves kRows rows per iteration with all loads issued before the stores. Kept
// indices come from shared memory (`rows` = the kept list) or from global
// memory (`rows` = kept_idx [B, k1]); an index outside 0..L-1 gives a zero row.
template <int VPL>
__device__ __forceinline__ void copy_rows(const uint4* __restrict__ y, int L, int Cv, int b,
                                          int k1, const int32_t* rows, bool rows_in_smem,
                                          int r_first, int r_step, uint4* __restrict__ y_kept) {
  const int lane = threadIdx.x & 31;
  constexpr int kRows = VPL >= 4 ? 1 : 4 / VPL;  // 16 registers of row data in flight
  for (int r0 = r_first; r0 < k1; r0 += r_step * kRows) {
    uint4 v[kRows][VPL];
#pragma unroll
    for (int j = 0; j < kRows; ++j) {
      const int r = r0 + r_step * j;
      if (r < k1) {
        const int t = rows_in_smem ? rows[r] : __ldg(rows + static_cast<size_t>(b) * k1 + r);
        if (t >= 0 && t < L) {
          const uint4* src = y + (static_cast<size_t>(b) * L + t) * Cv;
#pragma unroll
          for (int i = 0; i < VPL; ++i)
            if (lane + 32 * i < Cv) v[j][i] = __ldg(src + lane + 32 * i);
        } else {
#pragma unroll
          for (int i = 0; i < VPL; ++i) v[j][i] = make_uint4(0, 0, 0, 0);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kRows; ++j) {
      const int r = r0 + r_step * j;
      if (r < k1) {
        uint4* dst = y_kept + (static_cast<size_t>(b) * k1 + r) * Cv;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
          if (lane + 32 * i < Cv) __stcs(dst + lane + 32 * i, v[j][i]);
      }
    }
  }
}

// Fused: CTA (b, j0) of B x S selects sample b's kept rows and copies rows
// j0, j0 + S, ... of them; CTA (b, 0) also writes scores and kept_idx.
constexpr int kSelGatherThreads = 512;

// Two CTAs per SM, except for the widest rows (C > 1024), whose 32 registers of
// row data per lane need more than half of an SM's register file.
template <int VPL>
__global__ void __launch_bounds__(kSelGatherThreads, VPL >= 8 ? 1 : 2) select_gather_kernel(
    const float* __restrict__ partials, int NP, int L, int k, int dist, bool cls,
    const uint4* __restrict__ y, int Cv, int S, float* __restrict__ scores,
    int32_t* __restrict__ kept, uint4* __restrict__ y_kept) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ uint32_t s_warp[64], s_sel[8], s_rng[2];
  __shared__ __align__(16) uint32_t s_hist[768], s_cand[64];
  pdl_trigger();
  init_select_smem(s_hist, s_sel, s_rng, s_cand);
  pdl_wait();
  const int b = blockIdx.x / S, j0 = blockIdx.x % S;
  const bool writer = j0 == 0;
  const SelSmem s = carve(dyn, L, s_warp, s_hist, s_sel, s_rng, s_cand);
  load_keys(partials, NP, L, b, writer ? scores : nullptr, s, dist, cls ? 1 : 0);
  select_into_smem(L, k, s, cls);
  const int k1 = k + (cls ? 1 : 0);
  if (writer)
    for (int i = threadIdx.x; i < k1; i += blockDim.x)
      kept[static_cast<size_t>(b) * k1 + i] = s.kept[i];
  const int w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  copy_rows<VPL>(y, L, Cv, b, k1, s.kept, true, j0 + S * w, S * nw, y_kept);
}

// Standalone gather: the warps of the grid are shared out over the samples;
// a sample's warps take its kept rows round robin.
template <int VPL>
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ y, int L, int Cv,
                                                     const int32_t* __restrict__ kept, int k1,
                                                     int B, uint4* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = static_cast<int>((gridDim.x * blockDim.x) >> 5);
  const int per_sample = nw / B > 0 ? nw / B : 1;
  const int groups = nw / per_sample;
  for (int b = gw / per_sample; b < B && gw < groups * per_sample; b += groups)
    copy_rows<VPL>(y, L, Cv, b, k1, kept, false, gw % per_sample, per_sample, out);
}

// Keys (L, padded) and the kept list (at most k + 1 entries).
static size_t select_smem(int L, int k) {
  return static_cast<size_t>((L + 3) & ~3) * 4 + static_cast<size_t>(k + 1) * 4;
}

cudaError_t launch_select(const float* partials, int num_partials, int B, int L, int keep_k,
                          int dist, bool cls, float* scores, int32_t* kept_idx,
                          cudaStream_t stream, bool pdl) {
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(select_smem(RS_MAX_L, RS_MAX_L)));
  if (e != cudaSuccess) return e;
  int threads = ((L + 31) / 32) * 32;
  if (threads < 64) threads = 64;
  if (L > kRankMaxL) threads = 1024;
  return launch(select_kernel, B, threads, select_smem(L, keep_k), stream, pdl, partials,
                num_partials, L, keep_k, dist, cls, scores, kept_idx);
}

template <int VPL>
static cudaError_t launch_gather_t(const void* y, int B, int L, int Cv, const int32_t* kept_idx,
                                   int k1, void* y_kept, int blocks, cudaStream_t stream, bool pdl) {
  return launch(gather_kernel<VPL>, blocks, 256, 0, stream, pdl, static_cast<const uint4*>(y), L,
                Cv, kept_idx, k1, B, static_cast<uint4*>(y_kept));
}

cudaError_t launch_gather(const void* y, int B, int L, int C, const int32_t* kept_idx, int k1,
                          void* y_kept, int num_sms, cudaStream_t stream, bool pdl) {
  const int Cv = C / 8;
  if (k1 <= 0) return cudaSuccess;
  int blocks = (B * k1 + 7) / 8;
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  const int vpl = (Cv + 31) / 32;
  if (vpl <= 1) return launch_gather_t<1>(y, B, L, Cv, kept_idx, k1, y_kept, blocks, stream, pdl);
  if (vpl <= 2) return launch_gather_t<2>(y, B, L, Cv, kept_idx, k1, y_kept, blocks, stream, pdl);
  if (vpl <= 4) return launch_gather_t<4>(y, B, L, Cv, kept_idx, k1, y_kept, blocks, stream, pdl);
  return launch_gather_t<8>(y, B, L, Cv, kept_idx, k1, y_kept, blocks, stream, pdl);
}

template <int VPL>
static cudaError_t launch_sg_t(const float* partials, int NP, int L, int k, int dist, bool cls,
                               const void* y, int Cv, int B, int S, float* scores, int32_t* kept,
                               void* y_kept, cudaStream_t stream, bool pdl) {
  auto kern = select_gather_kernel<VPL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(select_smem(RS_MAX_L, RS_MAX_L)));
  if (e != cudaSuccess) return e;
  return launch(kern, B * S, kSelGatherThreads, select_smem(L, k), stream, pdl, partials, NP, L, k,
                dist, cls, static_cast<const uint4*>(y), Cv, S, scores, kept,
                static_cast<uint4*>(y_kept));
}

cudaError_t launch_select_gather(const float* partials, int num_partials, const void* y, int B,
                                 int L, int C, int keep_k, int dist, bool cls, float* scores,
                                 int32_t* kept_idx, void* y_kept, int num_sms,
                                 cudaStream_t stream, bool pdl) {
  // CTAs per sample: about one CTA per SM when B is small, one per sample otherwise;
  // where that leaves more than a tenth of the SMs without a CTA (B = 32 on 148 SMs:
  // 128 CTAs), two per SM instead, which the copy's memory parallelism repays
  const int k1 = keep_k + (cls ? 1 : 0);
  int S = num_sms / B;
  if (S >= 1 && 10 * B * S < 9 * num_sms && (C / 8 + 31) / 32 < 8) S = 2 * num_sms / B;
  if (S > k1) S = k1;
  if (S < 1) S = 1;
  const int Cv = C / 8;
  const int vpl = (Cv + 31) / 32;
  if (vpl <= 1)
    return launch_sg_t<1>(partials, num_partials, L, keep_k, dist, cls, y, Cv, B, S, scores,
                          kept_idx, y_kept, stream, pdl);
  if (vpl <= 2)
    return launch_sg_t<2>(partials, num_partials, L, keep_k, dist, cls, y, Cv, B, S, scores,
                          kept_idx, y_kept, stream, pdl);
  if (vpl <= 4)
    return launch_sg_t<4>(partials, num_partials, L, keep_k, dist, cls, y, Cv, B, S, scores,
                          kept_idx, y_kept, stream, pdl);
  return launch_sg_t<8>(partials, num_partials, L, keep_k, dist, cls, y, Cv, B, S, scores,
                        kept_idx, y_kept, stream, pdl);
}

}  // namespace rs
