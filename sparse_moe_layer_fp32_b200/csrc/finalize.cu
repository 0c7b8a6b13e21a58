// MoE finalize: weighted top-k un-permute, post-RMSNorm of the sandwich norm, residual add.
//
//   m[t]   = sum_j w[t][j] * y[inv[t][j]]              (FP32)
//   out[t] = bf16( residual[t] + m[t] / sqrt(mean(m[t]^2) + eps) * gamma )
//
// The pages name this step (vLLM PR "Day-0 support for Reflection's Beam-1.0", sections
// "Status" and "Remaining work": moe_finalize.cu, fused with the sandwich norms; news
// article "vLLM adds day-zero Reflection Beam serving": fused normalisation and residual
// kernels).  One CTA per token; every global access is a 16-byte vector (8 BF16), and a
// warp's accesses are contiguous, so the k row gathers of y stream at full HBM width.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace beam {

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
    f[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);  // a -> low half
  return *reinterpret_cast<const uint32_t*>(&h);
}

constexpr int kFinThreads = 128;

// The next sublayer's sandwich pre-norm, fused: x_next = bf16(out / sqrt(mean(out^2) + eps)
// * gamma), out being the BF16 values just written.  Disabled when x == nullptr.
struct NextNorm {
  uint16_t* x;
  const uint16_t* gamma;
  float eps;
};

// 1 / sqrt(sum / H + eps) of a per-thread partial sum, over the CTA (blockDim % 32 == 0).
__device__ __forceinline__ float block_rinv(float part, int H, float eps, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  __syncthreads();  // s_red may still be read from a previous reduction
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = part;
  __syncthreads();
  float tot = 0.0f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) tot += s_red[i];
  return 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
}

// Large batches: CTAs of 128 threads, several chunks per thread, the weighted sums kept in
// shared memory until the RMS is known; many CTAs per SM hide the gather latency.
template <bool PRE>
__global__ void __launch_bounds__(kFinThreads) finalize_wide_kernel(const uint16_t* __restrict__ y,
                                                               const float* __restrict__ w,
                                                               const int32_t* __restrict__ inv,
                                                               const uint16_t* residual,
                                                               const uint16_t* __restrict__ gamma, int H, int k,
                                                               float eps, uint16_t* out, NextNorm nn) {
  extern __shared__ float m_s[];  // [H]
  __shared__ int s_row[16];
  __shared__ float s_w[16];
  __shared__ float s_red[kFinThreads / 32];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = inv[static_cast<size_t>(t) * k + threadIdx.x];
    s_w[threadIdx.x] = w[static_cast<size_t>(t) * k + threadIdx.x];
  }
  __syncthreads();
  const int nchunks = H / 8;
  float ss = 0.0f;
  for (int c = threadIdx.x; c < nchunks; c += kFinThreads) {
    float acc[8] = {};
    for (int j0 = 0; j0 < k; j0 += 8) {  // up to 8 rows' chunks in flight (top-8: all of them)
      uint4 yv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < k) yv[j] = __ldg(reinterpret_cast<const uint4*>(y + static_cast<size_t>(s_row[j0 + j]) * H) + c);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j >= k) break;
        float f[8];
        unpack8(yv[j], f);
        const float wj = s_w[j0 + j];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      m_s[c * 8 + i] = acc[i];
      ss = fmaf(acc[i], acc[i], ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int i = 0; i < kFinThreads / 32; ++i) tot += s_red[i];
  const float rinv = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
  float ss2 = 0.0f;
  for (int c = threadIdx.x; c < nchunks; c += kFinThreads) {
    float r[8], g[8];
    unpack8(reinterpret_cast<const uint4*>(residual + static_cast<size_t>(t) * H)[c], r);  // out may alias residual
    unpack8(__ldg(reinterpret_cast<const uint4*>(gamma) + c), g);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = r[2 * i] + m_s[c * 8 + 2 * i] * rinv * g[2 * i];
      const float b = r[2 * i + 1] + m_s[c * 8 + 2 * i + 1] * rinv * g[2 * i + 1];
      o[i] = pack_bf16x2(a, b);
    }
    const uint4 ov = make_uint4(o[0], o[1], o[2], o[3]);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = ov;
    if constexpr (PRE) {  // keep the BF16 output for the next sublayer's pre-norm
      float f[8];
      unpack8(ov, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        m_s[c * 8 + i] = f[i];
        ss2 = fmaf(f[i], f[i], ss2);
      }
    }
  }
  if constexpr (PRE) {
    const float r2 = block_rinv(ss2, H, nn.eps, s_red);
    for (int c = threadIdx.x; c < nchunks; c += kFinThreads) {
      float g[8];
      unpack8(__ldg(reinterpret_cast<const uint4*>(nn.gamma) + c), g);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = pack_bf16x2(m_s[c * 8 + 2 * i] * r2 * g[2 * i], m_s[c * 8 + 2 * i + 1] * r2 * g[2 * i + 1]);
      reinterpret_cast<uint4*>(nn.x + static_cast<size_t>(t) * H)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Small batches: one CTA per token, its rows staged in shared memory by bulk copies (a
// handful of CTAs must move each token's k rows of y, so the loads go through the copy
// engine rather than per-thread loads).  The residual row and gamma (and the next gamma) do
// not depend on the GEMM and are copied before the wait for it; inv and w come from the
// routing, two launches back, and are read first.  The last warp only issues the copies (a
// thread that issues copies runs its warp's math several times slower afterwards); the
// other threads own 8-value chunks, and the weighted sums are recomputed from shared
// memory in each pass instead of being kept.
template <bool PRE>
__global__ void __launch_bounds__(1024) finalize_small_kernel(const uint16_t* __restrict__ y,
                                                              const float* __restrict__ w,
                                                              const int32_t* __restrict__ inv,
                                                              const uint16_t* residual,
                                                              const uint16_t* __restrict__ gamma, int H, int k,
                                                              float eps, uint16_t* out, NextNorm nn, uint32_t* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* ys = reinterpret_cast<uint16_t*>(smem);  // [k][H]
  uint16_t* rs = ys + static_cast<size_t>(k) * H;     // [H] residual row
  uint16_t* gs = rs + H;                              // [H] gamma
  uint16_t* ngs = gs + H;                             // [H] next gamma (PRE)
  __shared__ uint64_t bars[2];
  __shared__ int s_row[16];
  __shared__ float s_w[16];
  __shared__ float s_red[32];
  __shared__ int s_abort;
  const int t = blockIdx.x;
  const int nc = static_cast<int>(blockDim.x) - 32;  // compute threads; thread nc issues the copies
  const bool copier = static_cast<int>(threadIdx.x) == nc;
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = __ldcg(inv + static_cast<size_t>(t) * k + threadIdx.x);
    s_w[threadIdx.x] = __ldcg(w + static_cast<size_t>(t) * k + threadIdx.x);
  }
  __syncthreads();
  if (copier) {
    mbar_arrive_expect_tx(&bars[0], (PRE ? 3u : 2u) * row_bytes);
    bulk_load(rs, residual + static_cast<size_t>(t) * H, row_bytes, &bars[0]);  // out may alias residual
    bulk_load(gs, gamma, row_bytes, &bars[0]);
    if constexpr (PRE) bulk_load(ngs, nn.gamma, row_bytes, &bars[0]);
  }
  pdl_wait();
  pdl_trigger();
  if (copier) {
    mbar_arrive_expect_tx(&bars[1], static_cast<uint32_t>(k) * row_bytes);
    for (int j = 0; j < k; ++j)
      bulk_load(ys + static_cast<size_t>(j) * H, y + static_cast<size_t>(s_row[j]) * H, row_bytes, &bars[1]);
  }
  const bool ok0 = mbar_wait_bounded(&bars[0], 0, &s_abort);
  const bool ok1 = mbar_wait_bounded(&bars[1], 0, &s_abort);
  if (!(ok0 && ok1) && threadIdx.x == 0) atomicOr(err, kErrTimeoutEpilogue);
  __syncwarp();  // every lane left the polling loop on its own: reconverge before the math
  const int nchunks = H / 8;
  const int c0 = static_cast<int>(threadIdx.x) < nc ? static_cast<int>(threadIdx.x) : nchunks;  // copy warp: none
  // m[c] = sum_j w_j y_j over this chunk's 8 values, in slot order
  auto weighted = [&](int c, float (&m)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      float f[8];
      unpack8(reinterpret_cast<const uint4*>(ys + static_cast<size_t>(j) * H)[c], f);
      const float wj = s_w[j];
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = fmaf(wj, f[i], m[i]);
    }
  };
  auto out_chunk = [&](int c, float rinv, float (&m)[8]) -> uint4 {
    float r[8], g[8];
    unpack8(reinterpret_cast<const uint4*>(rs)[c], r);
    unpack8(reinterpret_cast<const uint4*>(gs)[c], g);
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = pack_bf16x2(r[2 * i] + m[2 * i] * rinv * g[2 * i], r[2 * i + 1] + m[2 * i + 1] * rinv * g[2 * i + 1]);
    return make_uint4(o[0], o[1], o[2], o[3]);
  };
  float ss = 0.0f;
  for (int c = c0; c < nchunks; c += nc) {
    float m[8];
    weighted(c, m);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(m[i], m[i], ss);
  }
  const float rinv = block_rinv(ss, H, eps, s_red);
  float ss2 = 0.0f;
  for (int c = c0; c < nchunks; c += nc) {
    float m[8];
    weighted(c, m);
    const uint4 ov = out_chunk(c, rinv, m);
    reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * H)[c] = ov;
    if constexpr (PRE) {  // the next pre-norm reads the BF16 values just written
      float f[8];
      unpack8(ov, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ss2 = fmaf(f[i], f[i], ss2);
    }
  }
  if constexpr (PRE) {
    const float r2 = block_rinv(ss2, H, nn.eps, s_red);
    for (int c = c0; c < nchunks; c += nc) {
      float m[8], f[8], g[8];
      weighted(c, m);
      unpack8(out_chunk(c, rinv, m), f);  // the same BF16 values as stored above
      unpack8(reinterpret_cast<const uint4*>(ngs)[c], g);
      uint32_t o[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(f[2 * i] * r2 * g[2 * i], f[2 * i + 1] * r2 * g[2 * i + 1]);
      reinterpret_cast<uint4*>(nn.x + static_cast<size_t>(t) * H)[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

static size_t finalize_small_smem(int H, int k) { return static_cast<size_t>(k + 3) * H * 2; }

template <bool PRE>
static cudaError_t launch_finalize_t(const uint16_t* y, const float* w, const int32_t* inv, const uint16_t* residual,
                                     const uint16_t* gamma, int T, int H, int k, float eps, uint16_t* out,
                                     NextNorm nn, uint32_t* err, cudaStream_t s, int form_T) {
  const int nchunks = H / 8;
  const size_t small = finalize_small_smem(H, k);
  if ((form_T > 0 ? form_T : T) < 256 && small <= 200 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(finalize_small_kernel<PRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(small));
    if (e != cudaSuccess) return e;
    const int threads = std::min(1024, ((nchunks + 31) / 32) * 32 + 32);  // + the copy warp
    return launch_pdl(finalize_small_kernel<PRE>, dim3(T), dim3(threads), small, s, y, w, inv, residual, gamma, H, k,
                      eps, out, nn, err);
  }
  const size_t smem = static_cast<size_t>(H) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(finalize_wide_kernel<PRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(finalize_wide_kernel<PRE>, dim3(T), dim3(kFinThreads), smem, s, y, w, inv, residual, gamma, H, k,
                    eps, out, nn);
}

cudaError_t launch_finalize(const uint16_t* y, const float* w, const int32_t* inv, const uint16_t* residual,
                            const uint16_t* gamma, int T, int H, int k, float eps, uint16_t* out, uint16_t* next_x,
                            const uint16_t* next_gamma, float next_eps, uint32_t* err, cudaStream_t s, int form_T) {
  const NextNorm nn{next_x, next_gamma, next_eps};
  if (next_x) return launch_finalize_t<true>(y, w, inv, residual, gamma, T, H, k, eps, out, nn, err, s, form_T);
  return launch_finalize_t<false>(y, w, inv, residual, gamma, T, H, k, eps, out, nn, err, s, form_T);
}

}  // namespace beam
