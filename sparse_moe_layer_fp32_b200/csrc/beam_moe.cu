// C ABI of libbeam_moe: handle, device memory, TMA descriptors and the forward sequence.
// The operation and its sources are described in include/beam_moe.h.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/beam_moe.h"
#include "common.cuh"
#include "internal.h"

using namespace beam;

struct beam_moe_ctx {
  beam_moe_config cfg;
  int H, E, k, I, Ip, Tmax;  // Ip: I rounded up to the K tile (the down GEMM's K)
  int64_t Rmax, nblk_max, n_chunks_max;
  int num_sms;
  // weights (owned, repacked)
  float* router_w;
  uint16_t* router_w3;  // BF16 split of router_w, tiled for the tensor-core router
  uint8_t *w_gu_tiles, *w_d_tiles;  // contiguous GEMM weight tiles (codes + scales)
  float *w_gu_alpha, *w_d_alpha;
  uint16_t* gamma;
  // workspace
  float* logits;
  int64_t logits_floats;
  int32_t *ids, *chunk_counts, *chunk_base, *offsets, *sf_block, *num_mblocks, *perm, *inv;
  int32_t* tile_row;  // [T][k]: 128 x activation block + row in it (where slot (t, j) goes in A1)
  float* w;
  MBlock* mblocks;
  uint8_t *a1, *a2;  // activation units: per 128-row block and K step, codes then scales
  uint16_t* y;
  uint32_t* err;
  unsigned int* route_counter;  // last-CTA election of the fused small-batch routing kernel
  uint32_t* sched;              // tile scheduler of the expert GEMM launch (sched_words(nblk_max))
  int32_t router_mode;          // BEAM_MOE_ROUTER_*: which router batches of more than 16 tokens use
  int32_t fmt;                  // BEAM_MOE_FMT_*: expert weight and activation format
  int kv;                       // K values per activation / weight tile: 256 (NVFP4), 128 (MXFP8)
  int act_unit;                 // bytes per 128-row block per K step: 16384 codes + 2048 scales
                                // (NVFP4) or + 512 (MXFP8)
  uint16_t *stage_x, *stage_res, *stage_out;
  // beam_moe_forward_host: the residual's upload runs on a second stream while the forward
  // computes; the finalize waits for it (created on the first host-buffer forward)
  cudaStream_t copy_stream;
  cudaEvent_t ev_start, ev_res;
  // ... and batches of 2 x host_chunk_tokens or more run in parts of host_chunk_tokens: part
  // c's output copies back on down_stream while later parts upload and compute
  int32_t host_chunk_tokens;
  cudaStream_t down_stream;
  cudaEvent_t ev_down;
  std::vector<cudaEvent_t> part_events;  // 3 per part: x landed, residual landed, finalized
  // tensor parallelism (beam_moe_tp_*): this handle holds one rank's slice of the experts
  uint8_t* tp_region;           // this rank's exchange region (owned), or null
  uint8_t** tp_regions_dev;     // device array [kMaxTpRanks]: every rank's region
  TpGroup tp;                   // every rank's region, this rank, the group size
  bool tp_attached;
  int tp_next_phase;            // the phase of beam_moe_forward_tp_phase that may run next (0..2)
  bool tp_two_shot;             // the forward in flight reduces in two steps
  int32_t tp_two_shot_min;      // from this batch size on (beam_moe_set_tp_two_shot_tokens)
  uint32_t tp_epoch;            // forwards so far in this group (the flag value of the last one)
  unsigned int* tp_counter;     // CTA arrivals of tp_partial [0] and of the two-shot tp_reduce [1]
  int tp_last_T;
  // expert parallelism (beam_moe_create_ep*): this handle holds experts [e_begin, e_begin + e_count)
  int e_begin, e_count;
  bool ep;
  int ep_next_phase;            // the phase of beam_moe_forward_ep_phase that may run next (0..3)
  int ep_T;                     // this rank's tokens in the current forward
  unsigned int* ep_counter;     // CTA arrivals of ep_combine
  EpLayout ep_lay;              // this rank's region (the same layout on every rank)
  EpDest* ep_dst;               // [E]: where this rank's rows of each expert go
  int32_t* ep_own_rows;         // rows this rank received in the current forward
  int32_t* inv_identity;        // [max_tokens k]: i, the returned rows' slot order
  int last_T;
  int last_splits;  // logits layout of the last forward: [splits][T][E] partial sums
  int last_launches;
  std::vector<void*> allocs;
  // optional per-kernel timing
  static constexpr int kMaxEvents = 17;
  bool profiling;
  bool profiled_last;
  cudaEvent_t events[kMaxEvents];
  const char* names[kMaxEvents];
};

namespace {

beam_moe_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return BEAM_MOE_OK;
  if (e == cudaErrorMemoryAllocation) return BEAM_MOE_ERR_OOM;
  return BEAM_MOE_ERR_CUDA;
}

#define BEAM_TRY(call)                              \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_status(e_);  \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D BF16 tensor [rows][cols]; boxes of 32 values (64 bytes) x box_rows, 64-byte swizzle.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
cudaError_t dalloc(beam_moe_ctx* h, T** p, size_t bytes) {
  void* q = nullptr;
  cudaError_t e = cudaMalloc(&q, std::max<size_t>(bytes, 16));
  if (e != cudaSuccess) return e;
  h->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return cudaSuccess;
}

void free_all(beam_moe_ctx* h) {
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
}

beam_moe_status check_shape(int H, int E, int k) {
  if (H <= 0 || E <= 0 || k <= 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (H % 256 != 0 || k > 16 || k > E || E > 1024 || (E >= 32 && E % 32 != 0)) return BEAM_MOE_ERR_UNSUPPORTED;
  return BEAM_MOE_OK;
}

int64_t route_ws_floats(int T, int H, int E) {
  return static_cast<int64_t>(router_split_count(T, H, E)) * T * E;
}

__global__ void store_f32_kernel(float* p, float v) { *p = v; }

// One CTA waits, with the kernels' bounded wait, on an mbarrier that nothing will complete.
__global__ void wait_timeout_probe_kernel(uint64_t limit_ns, uint32_t* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns)) atomicOr(err, kErrTimeoutMma);
}

// Kernels use 16-byte vector accesses on these pointers.
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Activation units (codes and scales) for a contraction of K values (multiple of kv).
size_t act_bytes(const beam_moe_ctx* h, int K) {
  return static_cast<size_t>(h->nblk_max) * (K / h->kv) * static_cast<size_t>(h->act_unit);
}

}  // namespace

extern "C" {

const char* beam_moe_status_string(beam_moe_status s) {
  switch (s) {
    case BEAM_MOE_OK: return "ok";
    case BEAM_MOE_ERR_INVALID_ARG: return "invalid argument";
    case BEAM_MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case BEAM_MOE_ERR_CUDA: return "CUDA runtime error";
    case BEAM_MOE_ERR_OOM: return "out of device memory";
    case BEAM_MOE_ERR_TIMEOUT: return "a bounded device wait timed out";
    case BEAM_MOE_ERR_DEVICE: return "device-side range check failed";
  }
  return "unknown status";
}

int64_t beam_moe_route_workspace_bytes(int32_t num_tokens, int32_t hidden, int32_t num_experts) {
  if (num_tokens <= 0 || hidden <= 0 || num_experts <= 0) return 0;
  return route_ws_floats(num_tokens, hidden, num_experts) * static_cast<int64_t>(sizeof(float));
}

}  // extern "C"

namespace {

// Weights of either format as create reads them (device pointers).
struct ExpertWeightsIn {
  const float* router_w;
  const uint8_t *w_gu, *w_gu_sf, *w_d, *w_d_sf;
  const float *w_gu_alpha, *w_d_alpha;  // NVFP4 only
  const uint16_t* gamma;
};

// e_count < 0: the handle holds every expert; else experts [e_begin, e_begin + e_count) of
// cfg->num_experts, whose weights (and tensor scales) are the arrays of wts.
beam_moe_status create_impl(const beam_moe_config* cfg, const ExpertWeightsIn& wts, int fmt, void* stream,
                            beam_moe_t* out, int e_begin = 0, int e_count = -1) {
  const bool mx = fmt == BEAM_MOE_FMT_MXFP8;
  const bool ep = e_count >= 0;
  if (!ep) e_count = cfg->num_experts;
  if (e_begin < 0 || e_count < 1 || e_begin > cfg->num_experts - e_count) return BEAM_MOE_ERR_INVALID_ARG;
  if (!wts.router_w || !wts.w_gu || !wts.w_gu_sf || !wts.w_d || !wts.w_d_sf || !wts.gamma)
    return BEAM_MOE_ERR_INVALID_ARG;
  if (!mx && (!wts.w_gu_alpha || !wts.w_d_alpha)) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned(wts.w_gu, 16) || !aligned(wts.w_d, 16) || !aligned(wts.gamma, 16)) return BEAM_MOE_ERR_INVALID_ARG;
  if (cfg->max_tokens <= 0 || !(cfg->rms_eps >= 0.0f)) return BEAM_MOE_ERR_INVALID_ARG;
  if (!mx && (!(cfg->alpha_a1 > 0.0f) || !(cfg->alpha_a2 > 0.0f))) return BEAM_MOE_ERR_INVALID_ARG;
  beam_moe_status st = check_shape(cfg->hidden, cfg->num_experts, cfg->top_k);
  if (st != BEAM_MOE_OK) return st;
  if (cfg->inter <= 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (cfg->inter % 128 != 0 || cfg->hidden > 16384) return BEAM_MOE_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(cfg->max_tokens) * cfg->top_k > (1ll << 30)) return BEAM_MOE_ERR_UNSUPPORTED;
  if (!tensor_map_encoder()) return BEAM_MOE_ERR_CUDA;

  beam_moe_ctx* h = new (std::nothrow) beam_moe_ctx();
  if (!h) return BEAM_MOE_ERR_OOM;
  h->cfg = *cfg;
  if (mx) h->cfg.alpha_a1 = h->cfg.alpha_a2 = 1.0f;  // MX activations carry no tensor scale
  h->fmt = fmt;
  h->ep = ep;
  h->e_begin = e_begin;
  h->e_count = e_count;
  h->kv = mx ? 128 : 256;
  h->act_unit = mx ? kActUnitMx : kActUnitNvfp4;
  h->H = cfg->hidden;
  h->E = cfg->num_experts;
  h->k = cfg->top_k;
  h->I = cfg->inter;
  h->Ip = (cfg->inter + h->kv - 1) / h->kv * h->kv;
  h->Tmax = cfg->max_tokens;
  h->Rmax = static_cast<int64_t>(h->Tmax) * h->k;
  h->nblk_max = (h->Rmax + 127) / 128 + h->E;
  h->n_chunks_max = (h->Tmax + kChunkTokens - 1) / kChunkTokens;
  h->last_T = 0;
  h->last_splits = 1;
  h->last_launches = 0;
  h->profiling = false;
  h->router_mode = BEAM_MOE_ROUTER_AUTO;
  h->tp_two_shot_min = BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS;
  h->host_chunk_tokens = BEAM_MOE_HOST_CHUNK_TOKENS;
  h->profiled_last = false;
  for (int i = 0; i < beam_moe_ctx::kMaxEvents; ++i) {
    h->events[i] = nullptr;
    h->names[i] = nullptr;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int H = h->H, E = h->E, I = h->I, Ip = h->Ip;

  auto fail = [&](cudaError_t e) {
    cudaStreamSynchronize(s);
    free_all(h);
    delete h;
    return cuda_status(e);
  };
#define CREATE_TRY(call)                    \
  do {                                      \
    cudaError_t e_ = (call);                \
    if (e_ != cudaSuccess) return fail(e_); \
  } while (0)

  int dev = 0;
  CREATE_TRY(cudaGetDevice(&dev));
  CREATE_TRY(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));

  // ---- weights
  CREATE_TRY(dalloc(h, &h->router_w, sizeof(float) * E * H));
  CREATE_TRY(dalloc(h, &h->router_w3, sizeof(uint16_t) * 3 * E * H));
  const int Ew = e_count;  // experts whose weights this handle holds
  const size_t tile_bytes = mx ? kMxTileBytes : kTileBytes;
  const size_t gu_tiles = static_cast<size_t>(Ew) * (2 * I / 256) * (H / h->kv);
  const size_t d_tiles = static_cast<size_t>(Ew) * (H / 256) * (Ip / h->kv);
  CREATE_TRY(dalloc(h, &h->w_gu_tiles, gu_tiles * tile_bytes));
  CREATE_TRY(dalloc(h, &h->w_d_tiles, d_tiles * tile_bytes));
  CREATE_TRY(dalloc(h, &h->w_gu_alpha, sizeof(float) * Ew));
  CREATE_TRY(dalloc(h, &h->w_d_alpha, sizeof(float) * Ew));
  CREATE_TRY(dalloc(h, &h->gamma, sizeof(uint16_t) * H));
  CREATE_TRY(cudaMemcpyAsync(h->router_w, wts.router_w, sizeof(float) * E * H, cudaMemcpyDeviceToDevice, s));
  CREATE_TRY(launch_split_router(h->router_w, E, H, h->router_w3, s));
  if (mx) {  // the accumulators need no dequantisation: unit scales in the block list
    const std::vector<float> ones(Ew, 1.0f);
    CREATE_TRY(cudaMemcpy(h->w_gu_alpha, ones.data(), sizeof(float) * Ew, cudaMemcpyHostToDevice));
    CREATE_TRY(cudaMemcpy(h->w_d_alpha, ones.data(), sizeof(float) * Ew, cudaMemcpyHostToDevice));
  } else {
    CREATE_TRY(cudaMemcpyAsync(h->w_gu_alpha, wts.w_gu_alpha, sizeof(float) * Ew, cudaMemcpyDeviceToDevice, s));
    CREATE_TRY(cudaMemcpyAsync(h->w_d_alpha, wts.w_d_alpha, sizeof(float) * Ew, cudaMemcpyDeviceToDevice, s));
  }
  CREATE_TRY(cudaMemcpyAsync(h->gamma, wts.gamma, sizeof(uint16_t) * H, cudaMemcpyDeviceToDevice, s));
  if (mx) {
    CREATE_TRY(launch_repack_tiles_mx(wts.w_gu, wts.w_gu_sf, Ew, 2 * I, H, I, h->w_gu_tiles, s));
    CREATE_TRY(launch_repack_tiles_mx(wts.w_d, wts.w_d_sf, Ew, H, I, 0, h->w_d_tiles, s));
  } else {
    CREATE_TRY(launch_repack_tiles(wts.w_gu, wts.w_gu_sf, Ew, 2 * I, H, H, I, h->w_gu_tiles, s));
    CREATE_TRY(launch_repack_tiles(wts.w_d, wts.w_d_sf, Ew, H, I, Ip, 0, h->w_d_tiles, s));
  }

  // ---- workspace
  int64_t lf = 0;
  for (int T = 1; T <= h->Tmax; T = (T < 64 ? T + 1 : T + 64)) lf = std::max(lf, route_ws_floats(T, H, E));
  lf = std::max(lf, route_ws_floats(h->Tmax, H, E));
  // the tensor-core router's partial logits: [splits][T][E] (every T: the split count steps)
  for (int T = 1; T <= h->Tmax; ++T)
    lf = std::max(lf, static_cast<int64_t>(router_tc_split_count(T, H, h->num_sms)) * T * E);
  for (int T = 1; T <= std::min(h->Tmax, kMaxSmallRouterTokens); ++T)
    if (route_small_supported(T, H, h->E, h->k)) lf = std::max(lf, route_small_ws_floats(T, H, h->E));
  h->logits_floats = lf;
  const int64_t R = h->Rmax;
  CREATE_TRY(dalloc(h, &h->logits, sizeof(float) * lf));
  CREATE_TRY(dalloc(h, &h->ids, sizeof(int32_t) * R));
  CREATE_TRY(dalloc(h, &h->w, sizeof(float) * R));
  CREATE_TRY(dalloc(h, &h->chunk_counts, sizeof(int32_t) * h->n_chunks_max * E));
  CREATE_TRY(dalloc(h, &h->chunk_base, sizeof(int32_t) * h->n_chunks_max * E));
  CREATE_TRY(dalloc(h, &h->offsets, sizeof(int32_t) * (E + 1)));
  CREATE_TRY(dalloc(h, &h->sf_block, sizeof(int32_t) * (E + 1)));
  CREATE_TRY(dalloc(h, &h->num_mblocks, sizeof(int32_t)));
  CREATE_TRY(dalloc(h, &h->mblocks, sizeof(MBlock) * h->nblk_max));
  CREATE_TRY(dalloc(h, &h->perm, sizeof(int32_t) * R));
  CREATE_TRY(dalloc(h, &h->inv, sizeof(int32_t) * R));
  CREATE_TRY(dalloc(h, &h->tile_row, sizeof(int32_t) * R));
  CREATE_TRY(dalloc(h, &h->a1, act_bytes(h, H)));
  CREATE_TRY(dalloc(h, &h->a2, act_bytes(h, Ip)));
  CREATE_TRY(dalloc(h, &h->y, sizeof(uint16_t) * static_cast<size_t>(R) * H));
  CREATE_TRY(dalloc(h, &h->err, sizeof(uint32_t)));
  CREATE_TRY(dalloc(h, &h->route_counter, sizeof(unsigned int)));
  CREATE_TRY(cudaMemsetAsync(h->route_counter, 0, sizeof(unsigned int), s));
  CREATE_TRY(dalloc(h, &h->sched, sizeof(uint32_t) * sched_words(h->nblk_max)));
  CREATE_TRY(dalloc(h, &h->stage_x, sizeof(uint16_t) * static_cast<size_t>(h->Tmax) * H));
  CREATE_TRY(dalloc(h, &h->stage_res, sizeof(uint16_t) * static_cast<size_t>(h->Tmax) * H));
  CREATE_TRY(dalloc(h, &h->stage_out, sizeof(uint16_t) * static_cast<size_t>(h->Tmax) * H));
  // The SwiGLU outputs beyond I (NVFP4 when I is not a multiple of 256) are never written:
  // their codes and scales must read as zero in the down GEMM.  The rows of a block past its
  // valid rows are also defined this way (they feed only accumulator rows never stored).
  CREATE_TRY(cudaMemsetAsync(h->a2, 0, act_bytes(h, Ip), s));
  CREATE_TRY(cudaMemsetAsync(h->a1, 0, act_bytes(h, H), s));
  CREATE_TRY(cudaMemsetAsync(h->err, 0, sizeof(uint32_t), s));
  if (ep) {
    if (E > 1024 || R >= (1ll << 24)) return fail(cudaErrorInvalidValue);  // the layout's limits
    CREATE_TRY(dalloc(h, &h->ep_dst, sizeof(EpDest) * E));
    CREATE_TRY(dalloc(h, &h->ep_own_rows, sizeof(int32_t)));
    CREATE_TRY(dalloc(h, &h->inv_identity, sizeof(int32_t) * R));
    std::vector<int32_t> iota(static_cast<size_t>(R));
    for (int64_t i = 0; i < R; ++i) iota[i] = static_cast<int32_t>(i);
    CREATE_TRY(cudaMemcpy(h->inv_identity, iota.data(), sizeof(int32_t) * R, cudaMemcpyHostToDevice));
    // the region: flag header, count matrix, arrival counters, origins, received activation
    // tiles and scales, returned rows
    size_t off = kTpHeaderBytes;
    auto take = [&](size_t bytes, size_t align) {
      off = (off + align - 1) / align * align;
      const size_t at = off;
      off += bytes;
      return at;
    };
    EpLayout& lay = h->ep_lay;
    lay.nblk = static_cast<int>(h->nblk_max);
    lay.rows = static_cast<int>(R);
    lay.counts = take(sizeof(int32_t) * kMaxTpRanks * E, 256);
    lay.arrivals = take(sizeof(uint32_t) * lay.nblk, 256);
    lay.origin = take(sizeof(int32_t) * R, 256);
    lay.a1 = take(act_bytes(h, H), 1024);
    lay.ret = take(sizeof(uint16_t) * static_cast<size_t>(R) * H, 1024);
    lay.bytes = (off + 255) / 256 * 256;
  }

  CREATE_TRY(cudaStreamSynchronize(s));
  CREATE_TRY(cudaGetLastError());
#undef CREATE_TRY
  *out = h;
  return BEAM_MOE_OK;
}

}  // namespace

extern "C" {

beam_moe_status beam_moe_create(const beam_moe_config* cfg, const beam_moe_weights* wts, void* stream,
                                beam_moe_t* out) {
  if (!cfg || !wts || !out) return BEAM_MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const ExpertWeightsIn in{wts->router_w, wts->w_gu, wts->w_gu_sf, wts->w_d, wts->w_d_sf,
                           wts->w_gu_alpha, wts->w_d_alpha, wts->gamma};
  return create_impl(cfg, in, BEAM_MOE_FMT_NVFP4, stream, out);
}

beam_moe_status beam_moe_create_mxfp8(const beam_moe_config* cfg, const beam_moe_weights_mxfp8* wts, void* stream,
                                      beam_moe_t* out) {
  if (!cfg || !wts || !out) return BEAM_MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const ExpertWeightsIn in{wts->router_w, wts->w_gu, wts->w_gu_sf, wts->w_d, wts->w_d_sf, nullptr, nullptr,
                           wts->gamma};
  return create_impl(cfg, in, BEAM_MOE_FMT_MXFP8, stream, out);
}

beam_moe_status beam_moe_create_ep(const beam_moe_config* cfg, const beam_moe_weights* wts, int32_t expert_begin,
                                   int32_t expert_count, void* stream, beam_moe_t* out) {
  if (!cfg || !wts || !out || expert_count < 1) return BEAM_MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const ExpertWeightsIn in{wts->router_w, wts->w_gu, wts->w_gu_sf, wts->w_d, wts->w_d_sf,
                           wts->w_gu_alpha, wts->w_d_alpha, wts->gamma};
  return create_impl(cfg, in, BEAM_MOE_FMT_NVFP4, stream, out, expert_begin, expert_count);
}

beam_moe_status beam_moe_create_ep_mxfp8(const beam_moe_config* cfg, const beam_moe_weights_mxfp8* wts,
                                         int32_t expert_begin, int32_t expert_count, void* stream, beam_moe_t* out) {
  if (!cfg || !wts || !out || expert_count < 1) return BEAM_MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const ExpertWeightsIn in{wts->router_w, wts->w_gu, wts->w_gu_sf, wts->w_d, wts->w_d_sf, nullptr, nullptr,
                           wts->gamma};
  return create_impl(cfg, in, BEAM_MOE_FMT_MXFP8, stream, out, expert_begin, expert_count);
}

int32_t beam_moe_expert_format(beam_moe_t h) { return h ? h->fmt : -1; }

beam_moe_status beam_moe_route(const void* x, const float* router_w, int32_t num_tokens, int32_t hidden,
                               int32_t num_experts, int32_t top_k, float* logits_ws, int32_t* ids, float* w,
                               void* stream) {
  beam_moe_status st = check_shape(hidden, num_experts, top_k);
  if (st != BEAM_MOE_OK) return st;
  if (num_tokens < 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens == 0) return BEAM_MOE_OK;
  if (!x || !router_w || !logits_ws || !ids || !w) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(logits_ws, 4) || !aligned(ids, 4) || !aligned(w, 4))
    return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BEAM_TRY(launch_router_logits(static_cast<const uint16_t*>(x), router_w, num_tokens, hidden, num_experts,
                                logits_ws, s));
  BEAM_TRY(launch_topk(logits_ws, router_split_count(num_tokens, hidden, num_experts), num_tokens, num_experts,
                       top_k, ids, w, s));
  return BEAM_MOE_OK;
}

// tp_phase: -1 the single-GPU forward; 0 the tensor-parallel forward up to the partial sums
// and their publication (tp_partial instead of finalize); 1 the all-reduce + finalize
// (tp_reduce) of the last phase 0: of every token (one-shot) or of this rank's slice
// (two-shot); 2 the gather of the other slices (two-shot; nothing in the one-shot form).  ep_phase (expert-parallel handles, tp_phase -1): 0 the
// routing of this rank's tokens and the count publication; 1 the layout and the dispatch; 2
// the expert GEMMs over the received rows and the combine; 3 the finalize of the returned
// rows (see expert_parallel.cu).
static beam_moe_status forward_impl(beam_moe_t h, const void* x, const void* residual, void* out, void* next_x,
                                    const void* next_gamma, float next_eps, int32_t num_tokens, void* stream,
                                    int tp_phase = -1, cudaEvent_t residual_ready = nullptr, int ep_phase = -1,
                                    int plan_T = 0, int plan_first = 0) {
  if (!h) return BEAM_MOE_ERR_INVALID_ARG;
  if (tp_phase < 0 && h->ep && ep_phase < 0) return BEAM_MOE_ERR_INVALID_ARG;  // holds only some experts
  if (tp_phase >= 0) {
    if (!h->tp_attached || h->ep) return BEAM_MOE_ERR_INVALID_ARG;
    if (tp_phase != h->tp_next_phase) return BEAM_MOE_ERR_INVALID_ARG;  // phases in order
    if (tp_phase > 0 && num_tokens != h->tp_last_T) return BEAM_MOE_ERR_INVALID_ARG;
  }
  if (num_tokens < 0 || num_tokens > h->Tmax) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens == 0) {
    h->last_T = 0;
    h->last_launches = 0;
    return BEAM_MOE_OK;
  }
  if (!x || !residual || !out) return BEAM_MOE_ERR_INVALID_ARG;
  if (x == out) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(residual, 16) || !aligned(out, 16)) return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = num_tokens, H = h->H, E = h->E, k = h->k;
  // Choices that change a row's arithmetic order (router form and slices, finalize form) and
  // the GEMM ring follow PT: a part of a larger batch (plan_T tokens, this part from token
  // plan_first on) computes that batch's bits.
  const int PT = plan_T > 0 ? plan_T : T;
  const int n_chunks = (T + kChunkTokens - 1) / kChunkTokens;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  int launches = 0;
  const bool prof = h->profiling;
  auto mark = [&](const char* name) -> cudaError_t {
    if (!prof) return cudaSuccess;
    h->names[launches] = name;
    return cudaEventRecord(h->events[launches + 1], s);
  };
  if (prof) BEAM_TRY(cudaEventRecord(h->events[0], s));
  auto finish = [&]() {
    h->last_T = T;
    h->last_launches = launches;
    h->profiled_last = prof;
    return BEAM_MOE_OK;
  };
  if (tp_phase == 1) {
    BEAM_TRY(launch_tp_reduce(static_cast<const uint16_t*>(residual), h->gamma, T, h->tp_two_shot, H, h->cfg.rms_eps,
                              h->tp, h->tp_epoch, static_cast<uint16_t*>(out), h->err, h->tp_counter + 1, s));
    BEAM_TRY(mark("tp_reduce"));
    ++launches;
    h->tp_next_phase = 2;
    return finish();
  }
  if (tp_phase == 2) {
    if (h->tp_two_shot) {
      BEAM_TRY(launch_tp_gather(T, H, h->tp, h->tp_epoch, static_cast<uint16_t*>(out), h->err, 4 * h->num_sms, s));
      BEAM_TRY(mark("tp_gather"));
      ++launches;
    }
    h->tp_next_phase = 0;
    return finish();
  }
  const BlockScales bscales{h->w_gu_alpha, h->w_d_alpha, h->cfg.alpha_a1, h->cfg.alpha_a2, h->e_begin,
                            h->e_begin + h->e_count};
  const bool mx = h->fmt == BEAM_MOE_FMT_MXFP8;
  // The expert GEMMs' arguments over a block list (this forward's, or the received rows')
  auto gemm_args = [&](const uint8_t* a1, int max_rows, const uint32_t* arrivals) {
    ExpertGemmArgs g{};
    g.mblocks = h->mblocks;
    g.num_mblocks = h->num_mblocks;
    g.max_rows_per_expert = max_rows;
    g.gu_n_tiles = h->I / 128;
    g.gu_k_tiles = H / h->kv;
    g.a1 = a1;
    g.w_gu = h->w_gu_tiles;
    g.a2 = h->a2;
    g.alpha_a2 = h->cfg.alpha_a2;
    g.d_n_tiles = H / 256;
    g.d_k_tiles = h->Ip / h->kv;
    g.w_d = h->w_d_tiles;
    g.y = h->y;
    g.y_cols = H;
    g.sched = h->sched;
    g.err = h->err;
    g.arrivals = arrivals;
    return g;
  };
  if (ep_phase >= 1) {
    const uint32_t epoch = h->tp_epoch + 1;  // the forward in flight
    uint8_t* region = h->tp_region;
    if (ep_phase == 1) {
      BEAM_TRY(launch_ep_layout(h->tp, h->ep_lay, E, bscales, h->mblocks, h->num_mblocks, h->sched,
                                static_cast<int>(sched_words(h->nblk_max)), h->ep_dst, h->ep_own_rows, epoch, h->err,
                                s));
      BEAM_TRY(mark("ep_layout"));
      ++launches;
      BEAM_TRY(launch_ep_dispatch(xb, h->ids, h->inv, h->offsets, h->ep_dst, T, H, k, h->fmt, h->cfg.alpha_a1, h->tp,
                                  h->ep_lay, s));
      BEAM_TRY(mark("ep_dispatch"));
      ++launches;
      return finish();
    }
    if (ep_phase == 2) {
      const ExpertGemmArgs g = gemm_args(region + h->ep_lay.a1, T * h->tp.world,
                                         reinterpret_cast<const uint32_t*>(region + h->ep_lay.arrivals));
      if (mx)
        BEAM_TRY(launch_gemm_experts_mx(g, h->num_sms, s));
      else
        BEAM_TRY(launch_gemm_experts(g, h->num_sms, s));
      BEAM_TRY(mark("gemm_experts"));
      ++launches;
      BEAM_TRY(launch_ep_combine(h->y, h->ep_own_rows, H, h->tp, h->ep_lay, epoch, h->ep_counter, 4 * h->num_sms, s));
      BEAM_TRY(mark("ep_combine"));
      ++launches;
      return finish();
    }
    // phase 3: this rank's tokens from their returned rows, in slot order
    BEAM_TRY(launch_ep_wait_returned(h->tp, epoch, h->err, s));
    BEAM_TRY(mark("ep_wait"));
    ++launches;
    BEAM_TRY(launch_finalize(reinterpret_cast<const uint16_t*>(region + h->ep_lay.ret), h->w, h->inv_identity,
                             static_cast<const uint16_t*>(residual), h->gamma, T, H, k, h->cfg.rms_eps,
                             static_cast<uint16_t*>(out), nullptr, nullptr, 0.0f, h->err, s));
    BEAM_TRY(mark("finalize"));
    ++launches;
    h->tp_epoch = epoch;
    return finish();
  }
  if (route_small_supported(PT, H, E, k)) {
    // router + top-k + histogram + scan + permutation in one launch
    int slices = 1;
    BEAM_TRY(launch_route_small(xb, h->router_w, T, H, E, k, h->logits, h->ids, h->w, h->offsets, h->sf_block,
                                h->mblocks, h->num_mblocks, h->perm, h->inv, h->tile_row, h->route_counter, h->sched,
                                static_cast<int>(sched_words(h->nblk_max)), bscales, h->err, &slices, s));
    BEAM_TRY(mark("route_small"));
    ++launches;
    h->last_splits = slices;
  } else {
    const bool simt_only = h->router_mode == BEAM_MOE_ROUTER_SIMT;
    // AUTO and TENSOR: slices of H whenever the split count is above one (measured faster than
    // one tile per CTA at every batch up to 32K tokens, and than the SIMT router from 17)
    const bool tc_split = !simt_only && router_tc_split_supported(H, E, k) && PT >= kRouterTcSplitMinTokens &&
                          router_tc_split_count(PT, H, h->num_sms) > 1;
    if (tc_split) {
      // tensor cores over (token tiles) x (slices of H), partial logits; the top-k kernel
      // sums the slices in order
      CUtensorMap map_x;
      const RouterTcPlan plan = router_tc_split_plan(PT, H, h->num_sms);
      if (!make_map_bf16(&map_x, xb, H, T, static_cast<uint32_t>(plan.tokens))) return BEAM_MOE_ERR_CUDA;
      const int splits = plan.splits;
      BEAM_TRY(launch_router_tc(map_x, plan.tokens, h->router_w3, T, H, E, k, h->logits, h->ids, h->w, h->err, s,
                                splits, plan_first));
      BEAM_TRY(mark("router_tc"));
      ++launches;
      h->last_splits = splits;
      BEAM_TRY(launch_topk(h->logits, splits, T, E, k, h->ids, h->w, s));
      BEAM_TRY(mark("topk"));
      ++launches;
    } else if (!simt_only && router_tc_supported(PT, H, E, k)) {
      // FP32-class logits on the tensor cores (BF16 x 3-part split), top-k in the epilogue
      CUtensorMap map_x;
      const int rt_tokens = router_tc_tokens_per_cta(PT, h->num_sms);
      if (!make_map_bf16(&map_x, xb, H, T, static_cast<uint32_t>(rt_tokens))) return BEAM_MOE_ERR_CUDA;
      BEAM_TRY(launch_router_tc(map_x, rt_tokens, h->router_w3, T, H, E, k, h->logits, h->ids, h->w, h->err, s, 1,
                                plan_first));
      BEAM_TRY(mark("router_tc"));
      ++launches;
      h->last_splits = 1;
    } else {
      BEAM_TRY(launch_router_logits(xb, h->router_w, T, H, E, h->logits, s));
      BEAM_TRY(mark("router"));
      ++launches;
      h->last_splits = router_split_count(T, H, E);
      BEAM_TRY(launch_topk(h->logits, h->last_splits, T, E, k, h->ids, h->w, s));
      BEAM_TRY(mark("topk"));
      ++launches;
    }
    BEAM_TRY(launch_chunk_hist(h->ids, T, k, E, h->chunk_counts, s));
    BEAM_TRY(mark("chunk_hist"));
    ++launches;
    BEAM_TRY(launch_scan(h->chunk_counts, n_chunks, E, h->chunk_base, h->offsets, h->sf_block, h->mblocks,
                         h->num_mblocks, h->sched, static_cast<int>(sched_words(h->nblk_max)), bscales, s));
    BEAM_TRY(mark("scan"));
    ++launches;
    BEAM_TRY(launch_scatter(h->ids, h->chunk_base, h->offsets, h->sf_block, T, k, E, h->perm, h->inv, h->tile_row,
                            s));
    BEAM_TRY(mark("scatter"));
    ++launches;
  }
  if (ep_phase == 0) {  // this rank's per-expert row counts to every rank
    BEAM_TRY(launch_ep_counts(h->offsets, E, h->tp, h->ep_lay, h->tp_epoch + 1, s));
    BEAM_TRY(mark("ep_counts"));
    ++launches;
    return finish();
  }
  if (mx)
    BEAM_TRY(launch_quant_a1_mx(xb, h->tile_row, T, H, k, h->a1, s));
  else
    BEAM_TRY(launch_quant_a1(xb, h->tile_row, T, H, k, h->cfg.alpha_a1, h->a1, s));
  BEAM_TRY(mark("quant_a1"));
  ++launches;

  // a token chooses an expert at most once: at most T rows per expert
  const ExpertGemmArgs g = gemm_args(h->a1, PT, nullptr);
  if (mx)
    BEAM_TRY(launch_gemm_experts_mx(g, h->num_sms, s));
  else
    BEAM_TRY(launch_gemm_experts(g, h->num_sms, s));
  BEAM_TRY(mark("gemm_experts"));
  ++launches;
  if (tp_phase == 0) {
    BEAM_TRY(launch_tp_partial(h->y, h->w, h->inv, h->ids, h->e_begin, h->e_begin + h->e_count, T, H, k, h->tp,
                               h->tp_epoch + 1, h->tp_counter, s));
    BEAM_TRY(mark("tp_partial"));
    ++launches;
    ++h->tp_epoch;
    h->tp_next_phase = 1;
    // two-shot only when every rank's slice of ceil(T / W) tokens holds one
    h->tp_two_shot = h->tp.world > 1 && T >= h->tp_two_shot_min &&
                     static_cast<int64_t>(tp_slice_tokens(T, h->tp.world)) * (h->tp.world - 1) < T;
    h->tp_last_T = T;
  } else {
    if (residual_ready) BEAM_TRY(cudaStreamWaitEvent(s, residual_ready, 0));
    BEAM_TRY(launch_finalize(h->y, h->w, h->inv, static_cast<const uint16_t*>(residual), h->gamma, T, H, k,
                             h->cfg.rms_eps, static_cast<uint16_t*>(out), static_cast<uint16_t*>(next_x),
                             static_cast<const uint16_t*>(next_gamma), next_eps, h->err, s, PT));
    BEAM_TRY(mark("finalize"));
    ++launches;
  }
  h->last_T = T;
  h->last_launches = launches;
  h->profiled_last = prof;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward(beam_moe_t h, const void* x, const void* residual, void* out, int32_t num_tokens,
                                 void* stream) {
  return forward_impl(h, x, residual, out, nullptr, nullptr, 0.0f, num_tokens, stream);
}

beam_moe_status beam_moe_forward_prenorm(beam_moe_t h, const void* x, const void* residual, void* out, void* next_x,
                                         const void* next_gamma, float next_eps, int32_t num_tokens, void* stream) {
  if (!h || num_tokens < 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens > 0) {
    if (!next_x || !next_gamma || !(next_eps >= 0.0f)) return BEAM_MOE_ERR_INVALID_ARG;
    if (!aligned(next_x, 16) || !aligned(next_gamma, 16)) return BEAM_MOE_ERR_INVALID_ARG;
    if (next_x == x || next_x == residual || next_x == out) return BEAM_MOE_ERR_INVALID_ARG;
  }
  return forward_impl(h, x, residual, out, next_x, next_gamma, next_eps, num_tokens, stream);
}

int64_t beam_moe_tp_region_bytes(beam_moe_t h) {
  if (!h) return 0;
  if (h->ep) return static_cast<int64_t>(h->ep_lay.bytes);
  const int64_t part = 2ll * h->Tmax * h->H * static_cast<int64_t>(sizeof(float));
  const int64_t rows = static_cast<int64_t>(h->Tmax) * h->H * static_cast<int64_t>(sizeof(uint16_t));
  return static_cast<int64_t>(kTpHeaderBytes) + part + rows;
}

beam_moe_status beam_moe_tp_region(beam_moe_t h, void** region) {
  if (!h || !region) return BEAM_MOE_ERR_INVALID_ARG;
  if (!h->tp_region) {
    // built into locals and published only when every step succeeded (a failed call leaves
    // the handle without a region; what it allocated is freed with the handle)
    const size_t bytes = static_cast<size_t>(beam_moe_tp_region_bytes(h));
    uint8_t* region = nullptr;
    uint8_t** table = nullptr;
    unsigned int *tp_counter = nullptr, *ep_counter = nullptr;
    BEAM_TRY(dalloc(h, &region, bytes));
    BEAM_TRY(dalloc(h, &tp_counter, 2 * sizeof(unsigned int)));
    BEAM_TRY(dalloc(h, &table, sizeof(uint8_t*) * kMaxTpRanks));
    BEAM_TRY(dalloc(h, &ep_counter, sizeof(unsigned int)));
    BEAM_TRY(cudaMemset(ep_counter, 0, sizeof(unsigned int)));
    BEAM_TRY(cudaMemset(region, 0, kTpHeaderBytes));
    if (h->ep) {  // received blocks' unused rows read as zero
      BEAM_TRY(cudaMemset(region + h->ep_lay.a1, 0, act_bytes(h, h->H)));
      BEAM_TRY(cudaMemset(region + h->ep_lay.arrivals, 0, sizeof(uint32_t) * h->ep_lay.nblk));
      BEAM_TRY(cudaMemset(region + h->ep_lay.origin, 0xFF, sizeof(int32_t) * h->ep_lay.rows));  // no source yet
    }
    BEAM_TRY(cudaMemset(tp_counter, 0, 2 * sizeof(unsigned int)));
    BEAM_TRY(cudaDeviceSynchronize());
    h->tp_region = region;
    h->tp_counter = tp_counter;
    h->tp_regions_dev = table;
    h->ep_counter = ep_counter;
  }
  *region = h->tp_region;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_tp_attach(beam_moe_t h, int32_t rank, int32_t world, void* const* regions, void* stream) {
  if (!h || !regions || world < 1 || world > kMaxTpRanks || rank < 0 || rank >= world) return BEAM_MOE_ERR_INVALID_ARG;
  if (!h->tp_region || regions[rank] != h->tp_region) return BEAM_MOE_ERR_INVALID_ARG;
  for (int q = 0; q < world; ++q)
    if (!regions[q] || !aligned(regions[q], 256)) return BEAM_MOE_ERR_INVALID_ARG;
  // expert parallelism: rank r holds experts [r E / W, (r + 1) E / W), every rank as many
  if (h->ep && (h->e_count * world != h->E || h->e_begin != rank * h->e_count)) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  BEAM_TRY(cudaMemset(h->tp_region, 0, kTpHeaderBytes));  // no epoch published yet in this group
  // CTA arrival counters restart (a forward that gave up on a wait may have left a count)
  BEAM_TRY(cudaMemset(h->tp_counter, 0, 2 * sizeof(unsigned int)));
  BEAM_TRY(cudaMemset(h->ep_counter, 0, sizeof(unsigned int)));
  BEAM_TRY(cudaDeviceSynchronize());
  uint8_t* table[kMaxTpRanks] = {};
  for (int q = 0; q < world; ++q) table[q] = static_cast<uint8_t*>(regions[q]);
  BEAM_TRY(cudaMemcpy(h->tp_regions_dev, table, sizeof(table), cudaMemcpyHostToDevice));
  TpGroup g{};
  g.regions = h->tp_regions_dev;
  g.own = h->tp_region;
  g.rank = rank;
  g.world = world;
  g.buf_floats = static_cast<size_t>(h->Tmax) * h->H;
  h->tp = g;
  h->tp_epoch = 0;
  h->tp_next_phase = 0;
  h->tp_two_shot = false;
  h->ep_next_phase = 0;
  h->tp_attached = true;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward_ep_phase(beam_moe_t h, const void* x, const void* residual, void* out,
                                          int32_t num_tokens, int32_t phase, void* stream) {
  if (!h || !h->ep || !h->tp_attached || phase < 0 || phase > 3) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens <= 0 || static_cast<int64_t>(num_tokens) * h->tp.world > h->Tmax) return BEAM_MOE_ERR_INVALID_ARG;
  if (!x || !residual || !out || !aligned(x, 16) || !aligned(residual, 16) || !aligned(out, 16))
    return BEAM_MOE_ERR_INVALID_ARG;
  if (phase != h->ep_next_phase || (phase > 0 && num_tokens != h->ep_T)) return BEAM_MOE_ERR_INVALID_ARG;
  beam_moe_status st = forward_impl(h, x, residual, out, nullptr, nullptr, 0.0f, num_tokens, stream, -1, nullptr,
                                    phase);
  if (st != BEAM_MOE_OK) return st;
  h->ep_T = num_tokens;
  h->ep_next_phase = (phase + 1) % 4;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward_ep(beam_moe_t h, const void* x, const void* residual, void* out,
                                    int32_t num_tokens, void* stream) {
  for (int phase = 0; phase < 4; ++phase) {
    beam_moe_status st = beam_moe_forward_ep_phase(h, x, residual, out, num_tokens, phase, stream);
    if (st != BEAM_MOE_OK) return st;
  }
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward_tp_phase(beam_moe_t h, const void* x, const void* residual, void* out,
                                          int32_t num_tokens, int32_t phase, void* stream) {
  if (phase < 0 || phase > 2) return BEAM_MOE_ERR_INVALID_ARG;
  if (h && h->ep) return BEAM_MOE_ERR_INVALID_ARG;  // expert-parallel handles: beam_moe_forward_ep
  if (!h || num_tokens <= 0) return num_tokens == 0 && h ? BEAM_MOE_OK : BEAM_MOE_ERR_INVALID_ARG;
  if (phase >= 1 && (!residual || !out || !aligned(residual, 16) || !aligned(out, 16)))
    return BEAM_MOE_ERR_INVALID_ARG;
  return forward_impl(h, x, residual, out, nullptr, nullptr, 0.0f, num_tokens, stream, phase);
}

beam_moe_status beam_moe_forward_tp(beam_moe_t h, const void* x, const void* residual, void* out,
                                    int32_t num_tokens, void* stream) {
  for (int phase = 0; phase < 3; ++phase) {
    beam_moe_status st = beam_moe_forward_tp_phase(h, x, residual, out, num_tokens, phase, stream);
    if (st != BEAM_MOE_OK || num_tokens == 0) return st;
  }
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ipc_export(const void* dev_ptr, void* handle_out) {
  if (!dev_ptr || !handle_out) return BEAM_MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t hd;
  BEAM_TRY(cudaIpcGetMemHandle(&hd, const_cast<void*>(dev_ptr)));
  static_assert(sizeof(hd) == BEAM_MOE_IPC_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle_out, &hd, sizeof(hd));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ipc_import(const void* handle, void** dev_ptr) {
  if (!handle || !dev_ptr) return BEAM_MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t hd;
  std::memcpy(&hd, handle, sizeof(hd));
  BEAM_TRY(cudaIpcOpenMemHandle(dev_ptr, hd, cudaIpcMemLazyEnablePeerAccess));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(cudaIpcCloseMemHandle(dev_ptr));
  return BEAM_MOE_OK;
}

constexpr size_t kMaxDirectOutBytes = 2u << 20;

// The host-buffer forward of a large batch in parts of host_chunk_tokens tokens.  The copy
// stream uploads x and then the residual of part 0, 1, ... in order; the caller's stream runs
// each part's forward once its x has landed (its finalize once its residual has); part c's
// output goes back on down_stream as soon as it is final, while later parts upload and
// compute.  Host-to-device copies are the bound at large batches (x and residual are 2 T H
// bytes each way), so the device-to-host copies and the compute now hide under them.  Every
// part runs with the whole batch's choices of router form and slices, finalize form and
// GEMM ring (plan_T), so the output has the same bits as one forward of the whole batch.
static beam_moe_status forward_host_parts(beam_moe_t h, const void* x_host, const void* residual_host,
                                          void* out_host, int32_t T, cudaStream_t s) {
  const int ct = h->host_chunk_tokens;
  const int parts = (T + ct - 1) / ct;
  if (!h->down_stream) {
    BEAM_TRY(cudaStreamCreateWithFlags(&h->down_stream, cudaStreamNonBlocking));
    BEAM_TRY(cudaEventCreateWithFlags(&h->ev_down, cudaEventDisableTiming));
  }
  while (h->part_events.size() < static_cast<size_t>(3 * parts)) {
    cudaEvent_t e;
    BEAM_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    h->part_events.push_back(e);
  }
  const size_t row = sizeof(uint16_t) * static_cast<size_t>(h->H);
  // the staging buffers are free once everything before this call on `s` is done (the
  // previous host forward's parts and copies back included: it ended by waiting for them)
  BEAM_TRY(cudaEventRecord(h->ev_start, s));
  BEAM_TRY(cudaStreamWaitEvent(h->copy_stream, h->ev_start, 0));
  BEAM_TRY(cudaStreamWaitEvent(h->down_stream, h->ev_start, 0));
  for (int c = 0; c < parts; ++c) {
    const size_t off = row * static_cast<size_t>(c) * ct, n = row * static_cast<size_t>(std::min(ct, T - c * ct));
    BEAM_TRY(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(h->stage_x) + off, static_cast<const uint8_t*>(x_host) + off,
                             n, cudaMemcpyHostToDevice, h->copy_stream));
    BEAM_TRY(cudaEventRecord(h->part_events[3 * c], h->copy_stream));
    BEAM_TRY(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(h->stage_res) + off,
                             static_cast<const uint8_t*>(residual_host) + off, n, cudaMemcpyHostToDevice,
                             h->copy_stream));
    BEAM_TRY(cudaEventRecord(h->part_events[3 * c + 1], h->copy_stream));
  }
  for (int c = 0; c < parts; ++c) {
    const int Tc = std::min(ct, T - c * ct);
    const size_t off = row * static_cast<size_t>(c) * ct, n = row * static_cast<size_t>(Tc);
    BEAM_TRY(cudaStreamWaitEvent(s, h->part_events[3 * c], 0));
    const beam_moe_status st = forward_impl(h, reinterpret_cast<uint8_t*>(h->stage_x) + off,
                                            reinterpret_cast<uint8_t*>(h->stage_res) + off,
                                            reinterpret_cast<uint8_t*>(h->stage_out) + off, nullptr, nullptr, 0.0f, Tc,
                                            s, -1, h->part_events[3 * c + 1], -1, T, c * ct);
    if (st != BEAM_MOE_OK) return st;
    BEAM_TRY(cudaEventRecord(h->part_events[3 * c + 2], s));
    BEAM_TRY(cudaStreamWaitEvent(h->down_stream, h->part_events[3 * c + 2], 0));
    BEAM_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + off, reinterpret_cast<uint8_t*>(h->stage_out) + off,
                             n, cudaMemcpyDeviceToHost, h->down_stream));
  }
  // the call's work on `s` ends with out_host complete
  BEAM_TRY(cudaEventRecord(h->ev_down, h->down_stream));
  BEAM_TRY(cudaStreamWaitEvent(s, h->ev_down, 0));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward_host(beam_moe_t h, const void* x_host, const void* residual_host, void* out_host,
                                      int32_t num_tokens, void* stream) {
  if (!h) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens < 0 || num_tokens > h->Tmax) return BEAM_MOE_ERR_INVALID_ARG;
  if (num_tokens == 0) return beam_moe_forward(h, nullptr, nullptr, nullptr, 0, stream);
  if (!x_host || !residual_host || !out_host) return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = sizeof(uint16_t) * static_cast<size_t>(num_tokens) * h->H;
  if (!h->copy_stream) {
    BEAM_TRY(cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
    BEAM_TRY(cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming));
    BEAM_TRY(cudaEventCreateWithFlags(&h->ev_res, cudaEventDisableTiming));
  }
  const int ct = h->host_chunk_tokens;
  if (ct > 0 && num_tokens >= 2 * ct && h->router_mode != BEAM_MOE_ROUTER_SIMT)
    return forward_host_parts(h, x_host, residual_host, out_host, num_tokens, s);
  // x first, at the full host-to-device bandwidth; the residual upload then starts (after
  // everything before it on `stream`, including the previous forward's finalize, which
  // read the staging buffer) and overlaps the routing and the expert GEMMs; only the
  // finalize waits for it
  BEAM_TRY(cudaMemcpyAsync(h->stage_x, x_host, bytes, cudaMemcpyHostToDevice, s));
  BEAM_TRY(cudaEventRecord(h->ev_start, s));
  BEAM_TRY(cudaStreamWaitEvent(h->copy_stream, h->ev_start, 0));
  BEAM_TRY(cudaMemcpyAsync(h->stage_res, residual_host, bytes, cudaMemcpyHostToDevice, h->copy_stream));
  BEAM_TRY(cudaEventRecord(h->ev_res, h->copy_stream));
  // A small out (kMaxDirectOutBytes) in page-locked memory that the device can address: the
  // finalize stores it there itself (over PCIe, while it computes), so no copy follows the
  // forward (decode8: 52.2 k vs 50.6 k tokens/s end to end).  Larger outs go back by the copy
  // engine, which moves them faster than the finalize's stores (spec1024: 1.038 vs 1.031 M);
  // pageable memory always does.
  void* out_dev = nullptr;
  if (bytes <= kMaxDirectOutBytes) {
    cudaPointerAttributes pa{};
    if (cudaPointerGetAttributes(&pa, out_host) != cudaSuccess)
      (void)cudaGetLastError();  // an unknown pointer is pageable memory here: clear and copy
    else if (pa.type == cudaMemoryTypeHost && pa.devicePointer && aligned(pa.devicePointer, 16))
      out_dev = pa.devicePointer;
  }
  beam_moe_status st = forward_impl(h, h->stage_x, h->stage_res, out_dev ? out_dev : h->stage_out, nullptr, nullptr,
                                    0.0f, num_tokens, stream, -1, h->ev_res);
  if (st != BEAM_MOE_OK) return st;
  if (!out_dev) BEAM_TRY(cudaMemcpyAsync(out_host, h->stage_out, bytes, cudaMemcpyDeviceToHost, s));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_quantize_nvfp4(const float* src, int64_t rows, int64_t cols, float alpha, uint8_t* codes,
                                        uint8_t* sf, float* alpha_out, void* stream) {
  if (rows < 0 || cols < 0 || cols % 16 != 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return BEAM_MOE_OK;
  if (!src || !codes || !sf) return BEAM_MOE_ERR_INVALID_ARG;
  if (!(alpha > 0.0f) && !alpha_out) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(codes, 8) || (alpha_out && !aligned(alpha_out, 4))) return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (alpha > 0.0f) {
    BEAM_TRY(launch_quantize_rows(src, rows, cols, alpha, nullptr, codes, sf, s));
    if (alpha_out) {
      store_f32_kernel<<<1, 1, 0, s>>>(alpha_out, alpha);
      BEAM_TRY(cudaGetLastError());
    }
    return BEAM_MOE_OK;
  }
  // alpha_out first holds amax (as FP32 bits), then the scale amax / 2688
  BEAM_TRY(launch_amax(src, rows * cols, alpha_out, s));
  BEAM_TRY(launch_quantize_rows(src, rows, cols, 0.0f, alpha_out, codes, sf, s));
  BEAM_TRY(launch_amax_to_alpha(alpha_out, s));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_quantize_mxfp8(const float* src, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* sf,
                                        void* stream) {
  if (rows < 0 || cols < 0 || cols % 32 != 0) return BEAM_MOE_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return BEAM_MOE_OK;
  if (!src || !codes || !sf) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(codes, 16)) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(launch_quantize_rows_mx(src, rows, cols, codes, sf, static_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_debug_copy(beam_moe_t h, int32_t which, void* dst, size_t bytes, size_t* size_out,
                                    void* stream) {
  if (!h) return BEAM_MOE_ERR_INVALID_ARG;
  const int64_t T = h->last_T, R = T * h->k;
  const void* src = nullptr;
  size_t n = 0;
  switch (which) {
    case BEAM_MOE_BUF_LOGITS: src = h->logits; n = sizeof(float) * h->last_splits * T * h->E; break;
    case BEAM_MOE_BUF_IDS: src = h->ids; n = sizeof(int32_t) * R; break;
    case BEAM_MOE_BUF_WEIGHTS: src = h->w; n = sizeof(float) * R; break;
    case BEAM_MOE_BUF_OFFSETS: src = h->offsets; n = sizeof(int32_t) * (h->E + 1); break;
    case BEAM_MOE_BUF_PERM: src = h->perm; n = sizeof(int32_t) * R; break;
    case BEAM_MOE_BUF_INV: src = h->inv; n = sizeof(int32_t) * R; break;
    case BEAM_MOE_BUF_SFBLOCK: src = h->sf_block; n = sizeof(int32_t) * (h->E + 1); break;
    case BEAM_MOE_BUF_A1: src = h->a1; n = act_bytes(h, h->H); break;
    case BEAM_MOE_BUF_A2: src = h->a2; n = act_bytes(h, h->Ip); break;
    case BEAM_MOE_BUF_Y: src = h->y; n = sizeof(uint16_t) * static_cast<size_t>(R) * h->H; break;
    default: return BEAM_MOE_ERR_INVALID_ARG;
  }
  if (T == 0) n = 0;
  if (size_out) *size_out = n;
  if (!dst || bytes == 0 || n == 0) return BEAM_MOE_OK;
  BEAM_TRY(cudaMemcpyAsync(dst, src, std::min(bytes, n), cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_check(beam_moe_t h, void* stream) {
  if (!h) return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BEAM_TRY(cudaStreamSynchronize(s));
  uint32_t err = 0;
  BEAM_TRY(cudaMemcpy(&err, h->err, sizeof(err), cudaMemcpyDeviceToHost));
  if (err == 0) return BEAM_MOE_OK;
  BEAM_TRY(cudaMemset(h->err, 0, sizeof(uint32_t)));
  if (err & (kErrTimeoutProducer | kErrTimeoutMma | kErrTimeoutEpilogue)) return BEAM_MOE_ERR_TIMEOUT;
  return BEAM_MOE_ERR_DEVICE;
}

int32_t beam_moe_last_launch_count(beam_moe_t h) { return h ? h->last_launches : 0; }

beam_moe_status beam_moe_debug_wait_timeout(beam_moe_t h, int64_t limit_ns, void* stream) {
  if (!h || limit_ns <= 0 || limit_ns > static_cast<int64_t>(kWaitLimitNs)) return BEAM_MOE_ERR_INVALID_ARG;
  wait_timeout_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns), h->err);
  BEAM_TRY(cudaGetLastError());
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_set_host_chunk_tokens(beam_moe_t h, int32_t tokens) {
  if (!h || tokens < 0 || tokens % 256 != 0) return BEAM_MOE_ERR_INVALID_ARG;
  h->host_chunk_tokens = tokens;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_set_tp_two_shot_tokens(beam_moe_t h, int32_t min_tokens) {
  if (!h || min_tokens < 1) return BEAM_MOE_ERR_INVALID_ARG;
  h->tp_two_shot_min = min_tokens;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_set_router_mode(beam_moe_t h, int32_t mode) {
  if (!h || mode < BEAM_MOE_ROUTER_AUTO || mode > BEAM_MOE_ROUTER_TENSOR) return BEAM_MOE_ERR_INVALID_ARG;
  h->router_mode = mode;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_profile_enable(beam_moe_t h, int32_t enable) {
  if (!h) return BEAM_MOE_ERR_INVALID_ARG;
  if (enable && !h->events[0])
    for (int i = 0; i < beam_moe_ctx::kMaxEvents; ++i) BEAM_TRY(cudaEventCreate(&h->events[i]));
  h->profiling = enable != 0;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_profile_read(beam_moe_t h, float* ms, int32_t capacity, int32_t* count) {
  if (!h || !count || (capacity > 0 && !ms)) return BEAM_MOE_ERR_INVALID_ARG;
  *count = h->profiled_last ? h->last_launches : 0;
  if (!h->profiled_last) return BEAM_MOE_OK;
  BEAM_TRY(cudaEventSynchronize(h->events[h->last_launches]));
  for (int i = 0; i < h->last_launches && i < capacity; ++i)
    BEAM_TRY(cudaEventElapsedTime(&ms[i], h->events[i], h->events[i + 1]));
  return BEAM_MOE_OK;
}

const char* beam_moe_kernel_name(beam_moe_t h, int32_t index) {
  if (!h || index < 0 || index >= h->last_launches) return nullptr;
  return h->names[index];
}

void beam_moe_destroy(beam_moe_t h) {
  if (!h) return;
  cudaDeviceSynchronize();
  for (int i = 0; i < beam_moe_ctx::kMaxEvents; ++i)
    if (h->events[i]) cudaEventDestroy(h->events[i]);
  if (h->copy_stream) {
    cudaEventDestroy(h->ev_start);
    cudaEventDestroy(h->ev_res);
    cudaStreamDestroy(h->copy_stream);
  }
  if (h->down_stream) {
    cudaEventDestroy(h->ev_down);
    cudaStreamDestroy(h->down_stream);
  }
  for (cudaEvent_t e : h->part_events) cudaEventDestroy(e);
  free_all(h);
  delete h;
}

}  // extern "C"
