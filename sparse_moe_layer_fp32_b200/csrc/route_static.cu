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
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the current CUDA context (never reused within a process), or false when no
// context is current.  A device reset destroys the context the module was loaded into; the
// next context gets a new id, and the array a new address.
bool current_context_id(unsigned long long* id) {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<GetCurrent>(a);
    get_id = reinterpret_cast<GetId>(b);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device.  It is looked up the first
// time a device is used, and again only if the device's context has changed since (after a
// device reset, say), so a stale address is never handed to a kernel.  In host code
// `g_route_scratch` names a host-side stand-in, not device memory, so the kernels must
// receive the address that cudaGetSymbolAddress returns.
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (!g_scratch_addr[dev] || !have_ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);  // makes the device's context current if none was
    if (e != cudaSuccess) return e;
    if (!current_context_id(&ctx)) return cudaErrorDeviceUninitialized;  // no context after the lookup
    g_scratch_addr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx;
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
