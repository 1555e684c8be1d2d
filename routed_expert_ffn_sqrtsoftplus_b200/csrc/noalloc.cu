// Routing without any device allocation, for callers that cannot call
// cudaMalloc (see moe_route_noalloc in include/moe.h).
//
// The routing step needs one scratch buffer: the approximate fp32 logits
// [T, E] that the logits kernel writes and the top-k kernel reads. Here that
// buffer is a file-scope __device__ array instead of handle-owned memory; the
// kernels themselves are the same ones moe_forward launches.
#include <mutex>

#include "../../include/moe.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) float g_route_logits_scratch[MOE_NOALLOC_MAX_LOGITS];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The host-side
// name of a __device__ array is only a stand-in, so the address is looked up
// once per device with cudaGetSymbolAddress and cached.
moe_status scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_logits_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_route_noalloc(const void* x, const void* router_w, const float* router_bias, int32_t T,
                                        int32_t hidden, int32_t n_routed, int32_t top_k, float route_scale,
                                        int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
  if (T < 0 || hidden <= 0 || hidden % 8 != 0 || n_routed <= 0 || top_k <= 0 || top_k > n_routed)
    return MOE_ERR_INVALID_ARG;
  if (!(route_scale > 0.f) || route_scale == INFINITY) return MOE_ERR_INVALID_ARG;
  if (n_routed > 512 || top_k > 32) return MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(T) * n_routed > MOE_NOALLOC_MAX_LOGITS) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (x == nullptr || router_w == nullptr || topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_INVALID_ARG;
  {
    // every buffer is read or written by the kernels on the current device
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    const void* bufs[] = {x, router_w, router_bias, topk_idx, topk_w};
    for (const void* p : bufs)
      if (p != nullptr && !moe::device_pointer_on(p, dev)) return MOE_ERR_INVALID_ARG;
  }
  float* z = nullptr;
  moe_status st = scratch_for_current_device(&z);
  if (st != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The logits kernel overwrites all T*E entries before the top-k kernel reads
  // them, so nothing left in the array by an earlier call is ever used.
  if (moe::launch_router_logits(x, router_w, router_bias, z, T, hidden, n_routed, s) != cudaSuccess ||
      moe::launch_topk_refine(z, x, router_w, router_bias, T, hidden, n_routed, top_k, route_scale, moe::kRefineDelta,
                              topk_idx, topk_w, nullptr, s) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
