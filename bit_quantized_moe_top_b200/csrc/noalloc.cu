// Routing entry point that allocates no device memory.
//
// Some callers cannot call cudaMalloc: a plugin or extension hosted by an
// inference framework that owns every byte of device memory, or a serving loop
// that must never hit the implicit device-wide synchronisation of
// cudaMalloc/cudaFree. For them, moe_route_topk_noalloc runs the layer's
// routing kernel (top-k softmax, per-expert counts and offsets) with its
// scratch (per-block expert histograms and bases, the finishing ticket and the
// status word) taken from one fixed array in device memory that is part of the
// library image, instead of a layer's workspace.
//
// The array holds kNoAllocScratchInts 32-bit words (196 KiB). Every GPU that
// loads the library keeps it until the process exits. Its size bounds the
// request: ceil(T / 16) * E <= 16384 (for example T <= 4096 with E = 64, or
// T <= 1024 with E = 256).
#include <mutex>

#include "../../include/moe_layer.h"
#include "kernels.h"

namespace moeq {
namespace {

constexpr int kNoAllocBlockEntries = 16384;  // token blocks x experts
constexpr int kNoAllocHeader = 1024;         // ticket, status, n_active, poffsets, active
constexpr int kNoAllocScratchInts = kNoAllocHeader + 3 * kNoAllocBlockEntries;

static __device__ __align__(256) int g_route_scratch[kNoAllocScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device; looked up once
// per device (with that device current) and cached.
cudaError_t scratch_for_current_device(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moeq

using namespace moeq;

extern "C" moe_status_t moe_route_topk_noalloc(const float* logits, int T, int E, int top_k, unsigned flags, int* idx,
                                               float* w, int* counts, int* offsets, void* cuda_stream) {
  if (!logits || !idx || !w || !counts || !offsets || T < 1 || E < 1 || E > kMaxExperts || top_k < 1 ||
      top_k > kMaxTopK || top_k > E || (flags & ~MOE_FLAG_NO_TOPK_RENORM))
    return MOE_ERR_INVALID_ARG;
  // token blocks of 16, counted in 64-bit so that no T overflows the check
  if (((long long)T + 15) / 16 * E > kNoAllocBlockEntries) return MOE_ERR_TOO_LARGE;
  int* s = nullptr;
  if (scratch_for_current_device(&s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // the finishing ticket and the status word must start at zero
  if (cudaMemsetAsync(s, 0, kNoAllocHeader * sizeof(int), st) != cudaSuccess) return MOE_ERR_CUDA;
  RouteArgs a{};
  a.logits = logits;
  a.T = T;
  a.E = E;
  a.k = top_k;
  a.renorm = (flags & MOE_FLAG_NO_TOPK_RENORM) ? 0 : 1;
  a.idx = idx;
  a.w = w;
  a.counts = counts;
  a.offsets = offsets;
  a.ticket = s + 0;
  a.status = reinterpret_cast<unsigned*>(s + 1);
  a.n_active = s + 2;
  a.poffsets = s + 64;
  a.active = s + 512;
  a.block_counts = s + kNoAllocHeader;
  a.block_base = s + kNoAllocHeader + kNoAllocBlockEntries;
  a.pblock_base = s + kNoAllocHeader + 2 * kNoAllocBlockEntries;
  return launch_route_topk(a, st, nullptr) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
