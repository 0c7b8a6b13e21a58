// Tensor-parallel MoE finalize fused with its all-reduce.
//
// With the experts split over W ranks along the intermediate size, rank r's expert
// outputs y_r are partial sums: the layer needs m = sum_r m_r, m_r = sum_j w_j y_r[inv_j],
// before the post-RMSNorm (vLLM PR "Day-0 support for Reflection's Beam-1.0", section
// "Status": Beam's TP all-reduce fused with the sandwich norms and the MoE finalize;
// recipe "reflection/Beam-1.0-501B-A23B", "NVFP4 with TP4 on Blackwell").  Two kernels:
//
//   tp_partial: m_r for every token, FP32, into this rank's exchange region; the last CTA
//               then writes the forward's epoch into this rank's flag slot of every rank's
//               region (release, system scope: the stores reach peers over NVLink).
//   tp_reduce:  each CTA waits (bounded, acquire) until every rank's flag holds the epoch,
//               reads the W partials of its token from the ranks' regions (ranks in order,
//               so every rank computes the same bits), then the same FP32 arithmetic as the
//               single-GPU finalize: out = bf16(residual + m / sqrt(mean(m^2) + eps) * gamma).
//
// One-shot all-reduce (small batches, where latency rules): every rank's tp_reduce reads all
// W partials of every token, W T H 4 bytes per rank.  Two-shot (large batches): rank r's
// tp_reduce covers only its slice of the tokens, [r S, (r + 1) S) with S = ceil(T / W), so
// it reads T H 4 bytes; it writes the finished BF16 rows to its own output and to its
// region's row buffer, and its last CTA publishes them (second flag set); then tp_gather
// waits for every rank's rows and copies the other slices into the output (T H 2 bytes
// read over the links).  Both forms do the same arithmetic per token, so their bits agree.
// Partial buffers are double-buffered by epoch parity: a rank overwrites buffer b only in
// epoch e + 2, after it has seen every peer's epoch e + 1 flag, which a peer sets only after
// it finished reading buffer b in epoch e.  The row buffer is single: a rank writes it in
// epoch e + 1 only after every peer published its epoch e + 1 partials, which a peer does
// only after its tp_gather of epoch e has completed (stream order).
//
// On one GPU the ranks can run one after the other: every rank's tp_partial first, then
// every rank's tp_reduce, then every rank's tp_gather, whose waits are then already
// satisfied; nothing waits on a kernel that is not running.
#include "common.cuh"
#include "internal.h"

namespace beam {

// Both kernels: one CTA per token; a thread's k (or W) row loads of one 8-value chunk are all
// in flight at once (tp_threads: how many threads share a row).
constexpr int kTpMaxThreads = 1024;
constexpr int kTpMaxK = 16;


__device__ __forceinline__ void unpack8_bf16(const uint4 v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
    f[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
  }
}

__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a -> low half
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float* tp_part(uint8_t* region, int buf, size_t buf_floats) {
  return reinterpret_cast<float*>(region + kTpHeaderBytes) + static_cast<size_t>(buf) * buf_floats;
}
__device__ __forceinline__ uint32_t* tp_flags(uint8_t* region) { return reinterpret_cast<uint32_t*>(region); }
// The finished BF16 rows of the two-shot form, after the two partial buffers.
__device__ __forceinline__ uint16_t* tp_rows(uint8_t* region, size_t buf_floats) {
  return reinterpret_cast<uint16_t*>(tp_part(region, 2, buf_floats));
}

// Bounded acquire wait (thread q < W: rank q's flag in slot base + q of this rank's region)
// until every flag holds the epoch; false (and the error word set) when a wait ran out.
// Every thread of the CTA calls it; the barrier orders every thread's later loads.
__device__ __forceinline__ bool tp_wait_flags(const TpGroup& g, int base, uint32_t epoch, uint32_t* err,
                                              int* s_ok) {
  if (threadIdx.x == 0) *s_ok = 1;
  __syncthreads();
  if (threadIdx.x < g.world) {
    const uint32_t* flag = tp_flags(g.own) + base + threadIdx.x;
    const uint64_t t0 = globaltimer_ns();
    // epochs only grow; compare modulo 2^32
    while (static_cast<int32_t>(ld_acquire_sys(flag) - epoch) < 0) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicOr(err, kErrTimeoutEpilogue);
        *s_ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  return *s_ok != 0;
}

__global__ void __launch_bounds__(kTpMaxThreads) tp_partial_kernel(const uint16_t* __restrict__ y,
                                                                   const float* __restrict__ w,
                                                                   const int32_t* __restrict__ inv,
                                                                   const int32_t* __restrict__ ids, int e_begin,
                                                                   int e_end, int H, int k, TpGroup g, uint32_t epoch,
                                                                   uint32_t* __restrict__ counter) {
  __shared__ int s_row[kTpMaxK];
  __shared__ float s_w[kTpMaxK];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < k) {
    // a slot whose expert this rank does not hold contributes nothing here (weight 0, any
    // valid row: its y row is not written by this rank)
    const size_t i = static_cast<size_t>(t) * k + threadIdx.x;
    const int e = ids[i];
    const bool held = e >= e_begin && e < e_end;
    s_row[threadIdx.x] = held ? inv[i] : 0;
    s_w[threadIdx.x] = held ? w[i] : 0.0f;
  }
  __syncthreads();
  float* part = tp_part(g.own, static_cast<int>(epoch & 1u), g.buf_floats) + static_cast<size_t>(t) * H;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float acc[8] = {};
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 yv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)  // 8 rows' chunks in flight before the first use
        yv[j] = j0 + j < k ? __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j0 + j]) * H) + c)
                           : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j >= k || s_w[j0 + j] == 0.0f) continue;  // unheld slots: the row may hold anything
        float f[8];
        unpack8_bf16(yv[j], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(s_w[j0 + j], f[i], acc[i]);
      }
    }
    reinterpret_cast<float4*>(part)[2 * c] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    reinterpret_cast<float4*>(part)[2 * c + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  // The barrier orders the CTA's partial stores before thread 0's release (cumulative);
  // the last arrival acquires every CTA's, and its system-scope release stores of the flag
  // carry all of them to the ranks that acquire the flag.
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t done = atom_add_acq_rel_gpu(counter, 1u);
    if (done == gridDim.x - 1) {  // every CTA's partials are written: publish them
      *counter = 0u;              // ready for the next forward (stream order)
      for (int q = 0; q < g.world; ++q) st_release_sys(tp_flags(g.regions[q]) + g.rank, epoch);
    }
  }
}

// Token t = tok_begin + blockIdx.x.  publish (two-shot): also store the row into this rank's
// row buffer, and the last CTA publishes the epoch in flag slot kTpRowSlot + rank of every
// rank's region.
__global__ void __launch_bounds__(kTpMaxThreads) tp_reduce_kernel(const uint16_t* residual,
                                                                  const uint16_t* __restrict__ gamma, int tok_begin,
                                                                  int H, float eps, TpGroup g, uint32_t epoch,
                                                                  uint16_t* out, uint32_t* err, int publish,
                                                                  uint32_t* __restrict__ counter) {
  extern __shared__ float m_s[];  // [H]
  __shared__ float s_red[kTpMaxThreads / 32];
  __shared__ const float* s_part[kMaxTpRanks];  // this token's row in every rank's buffer
  __shared__ int s_ok;
  const int t = tok_begin + static_cast<int>(blockIdx.x);
  const int buf = static_cast<int>(epoch & 1u);
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < g.world)
    s_part[threadIdx.x] = tp_part(g.regions[threadIdx.x], buf, g.buf_floats) + static_cast<size_t>(t) * H;
  // the waiting threads' acquires order every thread's partial loads below
  if (!tp_wait_flags(g, 0, epoch, err, &s_ok)) return;
  float ss = 0.0f;
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float m[8] = {};
    for (int q0 = 0; q0 < g.world; q0 += 4) {  // ranks in order: the same sum on every rank
      float4 v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (q0 + i < g.world) {
          const float4* p = reinterpret_cast<const float4*>(s_part[q0 + i]) + 2 * c;
          v[2 * i] = __ldcv(p);  // peers' memory: not cached, fetched again
          v[2 * i + 1] = __ldcv(p + 1);
        }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (q0 + i >= g.world) break;
        m[0] += v[2 * i].x; m[1] += v[2 * i].y; m[2] += v[2 * i].z; m[3] += v[2 * i].w;
        m[4] += v[2 * i + 1].x; m[5] += v[2 * i + 1].y; m[6] += v[2 * i + 1].z; m[7] += v[2 * i + 1].w;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m_s[c * 8 + i] = m[i];
      ss = fmaf(m[i], m[i], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) tot += s_red[i];
  const float rinv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float r[8], gm[8];
    unpack8_bf16(reinterpret_cast<const uint4*>(residual + static_cast<size_t>(t) * H)[c], r);  // out may alias
    unpack8_bf16(__ldg(reinterpret_cast<const uint4*>(gamma) + c), gm);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = bf16x2(r[2 * i] + m_s[c * 8 + 2 * i] * rinv * gm[2 * i],
                    r[2 * i + 1] + m_s[c * 8 + 2 * i + 1] * rinv * gm[2 * i + 1]);
    const uint4 row = make_uint4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = row;
    if (publish) reinterpret_cast<uint4*>(tp_rows(g.own, g.buf_floats) + static_cast<size_t>(t) * H)[c] = row;
  }
  if (publish) {  // same publication pattern as tp_partial
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t done = atom_add_acq_rel_gpu(counter, 1u);
      if (done == gridDim.x - 1) {
        *counter = 0u;
        for (int q = 0; q < g.world; ++q) st_release_sys(tp_flags(g.regions[q]) + kTpRowSlot + g.rank, epoch);
      }
    }
  }
}

// Two-shot, second step: once every rank published its rows (bounded wait), copy the rows
// of the other ranks' slices (rank q: [q S, min(T, (q + 1) S))) from their row buffers into
// this rank's output, 16 bytes per thread, grid-stride.
__global__ void __launch_bounds__(256) tp_gather_kernel(int T, int S, int H, TpGroup g, uint32_t epoch,
                                                        uint16_t* out, uint32_t* err) {
  __shared__ int s_ok;
  pdl_wait();
  pdl_trigger();
  if (!tp_wait_flags(g, kTpRowSlot, epoch, err, &s_ok)) return;
  const int own_begin = g.rank * S, own_end = min(T, own_begin + S);
  const int own_rows = own_end - own_begin;
  const int chunks = H / 8;
  const size_t total = static_cast<size_t>(T - own_rows) * chunks;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    int t = static_cast<int>(i / chunks);
    const int c = static_cast<int>(i - static_cast<size_t>(t) * chunks);
    if (t >= own_begin) t += own_rows;  // skip this rank's own slice
    const int q = t / S;
    const uint4* src = reinterpret_cast<const uint4*>(tp_rows(g.regions[q], g.buf_floats) + static_cast<size_t>(t) * H);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = __ldcv(src + c);  // peers' memory: not cached
  }
}

// One thread per 8-value chunk for small batches (few CTAs: the latency of one token's
// loads decides); 128 threads looping over the chunks once there are many tokens (many CTAs
// per SM keep more loads in flight; the wide finalize measured 96% of HBM this way).
constexpr int kTpWideTokens = 256, kTpWideThreads = 128;
static int tp_threads(int H, int tokens) {
  if (tokens >= kTpWideTokens) return kTpWideThreads;
  const int want = (H / 8 + 31) / 32 * 32;
  return want < kTpMaxThreads ? want : kTpMaxThreads;
}

cudaError_t launch_tp_partial(const uint16_t* y, const float* w, const int32_t* inv, const int32_t* ids, int e_begin,
                              int e_end, int T, int H, int k, const TpGroup& g, uint32_t epoch, unsigned int* counter,
                              cudaStream_t s) {
  return launch_pdl(tp_partial_kernel, dim3(T), dim3(tp_threads(H, T)), 0, s, y, w, inv, ids, e_begin, e_end, H, k, g,
                    epoch, counter);
}

int tp_slice_tokens(int T, int world) { return (T + world - 1) / world; }

cudaError_t launch_tp_reduce(const uint16_t* residual, const uint16_t* gamma, int T, bool two_shot, int H, float eps,
                             const TpGroup& g, uint32_t epoch, uint16_t* out, uint32_t* err, unsigned int* counter,
                             cudaStream_t s) {
  const size_t smem = static_cast<size_t>(H) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(tp_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  int begin = 0, count = T;
  if (two_shot) {  // this rank's slice; the host only picks the two-shot form when every slice is non-empty
    const int S = tp_slice_tokens(T, g.world);
    begin = g.rank * S;
    count = min(T, begin + S) - begin;
    if (count <= 0) return cudaErrorInvalidValue;
  }
  // threads from the batch, not the slice: both forms then sum each row's squares in the
  // same order and give the same bits
  return launch_pdl(tp_reduce_kernel, dim3(count), dim3(tp_threads(H, T)), smem, s, residual, gamma, begin, H, eps, g,
                    epoch, out, err, two_shot ? 1 : 0, counter);
}

cudaError_t launch_tp_gather(int T, int H, const TpGroup& g, uint32_t epoch, uint16_t* out, uint32_t* err, int grid,
                             cudaStream_t s) {
  return launch_pdl(tp_gather_kernel, dim3(grid), dim3(256), 0, s, T, tp_slice_tokens(T, g.world), H, g, epoch, out,
                    err);
}

}  // namespace beam
