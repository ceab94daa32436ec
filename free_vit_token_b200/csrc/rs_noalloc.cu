// rs_noalloc.cu -- rs_ln_fc1_gelu_noalloc: the LayerNorm + fc1 + GELU step of
// rs_ln_fc1_gelu for callers that cannot allocate device memory when they call:
// a framework that owns every byte of device memory through its own pool and
// allows no other allocation, or latency-bound code that cannot afford a
// cudaMalloc or cudaFree, which may synchronise the whole device. Its scratch --
// the per-row LN statistics, the LN-folded fc1 weights and a status slot -- lives
// in one file-scope static device array instead of the library workspace. Every
// GPU that loads the library holds that array (kScratchBytes, about 8.6 MiB)
// until the process exits.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "rs.h"
#include "rs_internal.h"

namespace {

constexpr int64_t kMaxRows = 65536;        // M limit: LN statistics, 8 B per row
constexpr int64_t kMaxWeights = 4194304;   // H * C limit: folded weights, bf16
constexpr size_t kOffStats = 0;
constexpr size_t kOffWg = kOffStats + kMaxRows * 8;
constexpr size_t kOffG = kOffWg + kMaxWeights * 2;
constexpr size_t kOffC = kOffG + RS_MAX_H * 4;
constexpr size_t kOffErr = kOffC + RS_MAX_H * 4;
constexpr size_t kScratchBytes = kOffErr + 256;

// The scratch. In host code this name is only a host-side stand-in: the kernels
// get the device address from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch_ptr[kMaxDevices];  // device address of the array, per device
int g_num_sms[kMaxDevices];

// Once per device, with that device current: resolve the array's device address.
int setup(int dev) {
  if (g_scratch_ptr[dev] != nullptr) return RS_OK;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  g_num_sms[dev] = sms;
  g_scratch_ptr[dev] = static_cast<unsigned char*>(ptr);
  return RS_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace rs {

int noalloc_take_error() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RS_ERR_CUDA;
  unsigned char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    scratch = g_scratch_ptr[dev];
  }
  if (scratch == nullptr) return RS_OK;  // never called on this device: nothing recorded
  int v = 0;
  if (cudaMemcpy(&v, scratch + kOffErr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  if (v != 0 && cudaMemset(scratch + kOffErr, 0, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  return v;
}

}  // namespace rs

extern "C" int rs_ln_fc1_gelu_noalloc(const void* x, int M, int C, int H, const void* W1,
                                      const void* b1, const void* gamma, const void* beta,
                                      void* hidden, void* stream) {
  if (C < 64 || C > RS_MAX_C || C % 64 != 0 || H < 64 || H > RS_MAX_H || H % 64 != 0 || M < 0)
    return RS_ERR_SHAPE;
  // the scratch limits
  if (M > kMaxRows || static_cast<int64_t>(H) * C > kMaxWeights) return RS_ERR_SHAPE;
  if (M == 0) return RS_OK;
  if (!x || !W1 || !b1 || !gamma || !beta || !hidden) return RS_ERR_NULL;
  if (!aligned16(x) || !aligned16(W1) || !aligned16(b1) || !aligned16(gamma) ||
      !aligned16(beta) || !aligned16(hidden))
    return RS_ERR_ALIGN;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RS_ERR_CUDA;
  unsigned char* scratch = nullptr;
  int num_sms = 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const int s = setup(dev);
    if (s != RS_OK) return s;
    scratch = g_scratch_ptr[dev];
    num_sms = g_num_sms[dev];
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* stats = reinterpret_cast<float*>(scratch + kOffStats);
  void* wg = scratch + kOffWg;
  float* colg = reinterpret_cast<float*>(scratch + kOffG);
  float* colc = reinterpret_cast<float*>(scratch + kOffC);
  int* err = reinterpret_cast<int*>(scratch + kOffErr);

  if (rs::launch_ln_stats(x, M, C, stats, num_sms, st) != cudaSuccess) return RS_ERR_CUDA;
  if (rs::launch_ln_fold(W1, gamma, beta, b1, H, C, wg, colg, colc, num_sms, st) != cudaSuccess)
    return RS_ERR_CUDA;
  const int bn = rs::fc1_block_n(H);
  CUtensorMap tmX, tmW, tmHid;
  // single-CTA tiles: the B box holds all bn rows (rs::gemm_b_box_rows(bn, false))
  if (rs::make_tmap(&tmX, x, C, M, 128) != RS_OK ||
      rs::make_tmap(&tmW, wg, C, H, rs::gemm_b_box_rows(bn, false)) != RS_OK ||
      rs::make_tmap(&tmHid, hidden, H, M, rs::kEpiBoxRows, rs::fc1_out_box_cols(H, C, false)) !=
          RS_OK)
    return RS_ERR_CUDA;
  rs::MlpParams p{};
  p.M = M;
  p.N = H;
  p.K = C;
  p.n_blocks = H / bn;
  p.num_tiles = rs::gemm_num_tiles(M, p.n_blocks, /*pair=*/false);
  p.stats = reinterpret_cast<const float2*>(stats);
  p.colG = colg;
  p.colC = colc;
  p.out = static_cast<__nv_bfloat16*>(hidden);
  p.err = err;
  p.timeout_ns = rs::kDefaultTimeoutNs;
  p.debug_skip_kb = -1;
  if (rs::launch_fc1(tmX, tmW, tmHid, p, bn, false, /*pair=*/false, num_sms, st) != cudaSuccess) {
    cudaGetLastError();
    return RS_ERR_CUDA;
  }
  return RS_OK;
}
