// Routing (router logits + top-k + renormalise) for callers that cannot allocate device
// memory: the logits scratch is a fixed array compiled into this library instead of a
// caller- or handle-owned buffer.  Same kernels, same arithmetic as beam_moe_route.
#include <mutex>

#include "../../include/beam_moe.h"
#include "common.cuh"
#include "internal.h"

using namespace beam;

namespace {

// 2 Mi floats (8 MiB).  Every GPU that loads this library holds this array until the
// process exits.  It is shared by every call on that GPU and keeps the last call's
// contents.  The router kernels overwrite every element they later read, so nothing in it
// needs clearing between calls.
constexpr int64_t kStaticScratchFloats = int64_t(1) << 21;
static __device__ __align__(256) float g_route_scratch[kStaticScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device.
// In host code `g_route_scratch` names a host-side stand-in, not device memory, so the
// kernels must receive the address that cudaGetSymbolAddress returns.
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" beam_moe_status beam_moe_route_static(const void* x, const float* router_w, int32_t num_tokens,
                                                 int32_t hidden, int32_t num_experts, int32_t top_k, int32_t* ids,
                                                 float* w, void* stream) {
  if (hidden <= 0 || num_experts <= 0 || top_k <= 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (hidden % 256 != 0 || top_k > 16 || top_k > num_experts || num_experts > 1024 ||
      (num_experts >= 32 && num_experts % 32 != 0))
    return BEAM_MOE_ERR_UNSUPPORTED;
  if (num_tokens < 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens == 0) return BEAM_MOE_OK;
  if (!x || !router_w || !ids || !w) return BEAM_MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(router_w) & 15) ||
      (reinterpret_cast<uintptr_t>(ids) & 3) || (reinterpret_cast<uintptr_t>(w) & 3))
    return BEAM_MOE_ERR_INVALID_ARG;
  // The logits (possibly as partial sums over slices of H) must fit the fixed array.
  const int splits = router_split_count(num_tokens, hidden, num_experts);
  if (static_cast<int64_t>(splits) * num_tokens * num_experts > kStaticScratchFloats)
    return BEAM_MOE_ERR_UNSUPPORTED;
  float* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = launch_router_logits(static_cast<const uint16_t*>(x), router_w, num_tokens, hidden, num_experts, scratch, s);
  if (e != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  e = launch_topk(scratch, splits, num_tokens, num_experts, top_k, ids, w, s);
  if (e != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  return BEAM_MOE_OK;
}
