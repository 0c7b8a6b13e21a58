// Router of the MoE layer: FP32 logits = x W_r^T, then softmax / top-k / renormalise.
//
// The pages name a router GEMM for hidden 5120 -> 256 experts (vLLM PR "Day-0 support for
// Reflection's Beam-1.0", section "Status") and a specialised FP32 router kernel (news
// article "vLLM adds day-zero Reflection Beam serving", section "Agents worked on the
// serving path"); 8 of 256 experts per token (recipe "reflection/Beam-1.0-501B-A23B",
// section "Overview").
//
// Two logits kernels, both FP32 FFMA with BF16 x widened exactly to FP32:
//  * few tokens (decode): one CTA per expert streams its 20 KB weight row once and
//    dots it with every token; the bound is reading W_r (E*H*4 bytes) from HBM.
//  * many tokens: a 64x64-tiled SGEMM, split along H when there are too few tiles to
//    fill the GPU; the split partial sums are added in a fixed order by the top-k
//    kernel, so results are deterministic.
// These serve beam_moe_route and BEAM_MOE_ROUTER_SIMT; the layer's default router for
// batches above 16 tokens is the tensor-core one (router_tc.cu), whose partial logits the
// same top-k kernel sums.
// Top-k: one warp per token, E/32 logits per lane, k rounds of a warp arg-max
// (larger logit first, equal logits -> lower expert index).  Since softmax is monotone
// the top-k of p is the top-k of the logits, and p_j / sum_chosen p = softmax over the
// chosen logits, so the 256-way sum is not needed.
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace beam {

// ------------------------------------------------------------------ few tokens
__global__ void __launch_bounds__(256) router_gemv_kernel(const uint16_t* __restrict__ x,
                                                          const float* __restrict__ w, int T, int H, int E,
                                                          float* __restrict__ logits) {
  const int e = blockIdx.x;
  const float4* wr = reinterpret_cast<const float4*>(w + static_cast<size_t>(e) * H);
  float acc[kMaxSmallRouterTokens];
#pragma unroll
  for (int t = 0; t < kMaxSmallRouterTokens; ++t) acc[t] = 0.0f;
  const int n4 = H / 4;
  for (int c = threadIdx.x; c < n4; c += blockDim.x) {
    const float4 wv = __ldg(wr + c);
#pragma unroll
    for (int t = 0; t < kMaxSmallRouterTokens; ++t) {
      if (t < T) {
        const uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + static_cast<size_t>(t) * H) + c);
        acc[t] = fmaf(bf16_bits_to_f32(xv.x & 0xFFFFu), wv.x, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.x >> 16), wv.y, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.y & 0xFFFFu), wv.z, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.y >> 16), wv.w, acc[t]);
      }
    }
  }
  __shared__ float part[8][kMaxSmallRouterTokens];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < kMaxSmallRouterTokens; ++t) {
    float v = acc[t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) part[warp][t] = v;
  }
  __syncthreads();
  if (threadIdx.x < T) {
    float v = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) v += part[i][threadIdx.x];
    logits[static_cast<size_t>(threadIdx.x) * E + e] = v;
  }
}

// ------------------------------------------------------------------ many tokens
constexpr int RBM = 64, RBN = 64, RBK = 32;

// partial[split][T][E] = sum over this split's H range of x[t][h] * w[e][h]
__global__ void __launch_bounds__(256) router_sgemm_kernel(const uint16_t* __restrict__ x,
                                                           const float* __restrict__ w, int T, int H, int E,
                                                           int k_per_split, float* __restrict__ partial) {
  __shared__ __align__(16) float As[RBK][RBM + 4];
  __shared__ __align__(16) float Bs[RBK][RBN + 4];
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int m0 = blockIdx.y * RBM, n0 = blockIdx.x * RBN;
  const int split = blockIdx.z;
  const int kbeg = split * k_per_split, kend = kbeg + k_per_split;
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  const int lrow = tid >> 2, lk = (tid & 3) * 8;
  for (int k0 = kbeg; k0 < kend; k0 += RBK) {
    {  // x tile: 64 rows x 32 k, 8 BF16 per thread
      const int m = m0 + lrow;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (m < T) v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * H + k0 + lk));
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        As[lk + 2 * i][lrow] = bf16_bits_to_f32(u[i] & 0xFFFFu);
        As[lk + 2 * i + 1][lrow] = bf16_bits_to_f32(u[i] >> 16);
      }
    }
    {  // w tile: 64 experts x 32 k, 8 FP32 per thread
      const int n = n0 + lrow;
      float4 a = make_float4(0, 0, 0, 0), b = a;
      if (n < E) {
        const float4* p = reinterpret_cast<const float4*>(w + static_cast<size_t>(n) * H + k0 + lk);
        a = __ldg(p);
        b = __ldg(p + 1);
      }
      Bs[lk + 0][lrow] = a.x; Bs[lk + 1][lrow] = a.y; Bs[lk + 2][lrow] = a.z; Bs[lk + 3][lrow] = a.w;
      Bs[lk + 4][lrow] = b.x; Bs[lk + 5][lrow] = b.y; Bs[lk + 6][lrow] = b.z; Bs[lk + 7][lrow] = b.w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < RBK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = partial + static_cast<size_t>(split) * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < E) out[static_cast<size_t>(m) * E + n] = acc[i][j];
    }
  }
}

int router_split_count(int T, int H, int E) {
  if (T <= kMaxSmallRouterTokens) return 1;
  const int tiles = ((T + RBM - 1) / RBM) * ((E + RBN - 1) / RBN);
  int splits = 1;
  const int kblocks = H / RBK;
  while (tiles * splits < 2 * 148 && splits < 8 && kblocks % (splits * 2) == 0) splits *= 2;
  return splits;
}

cudaError_t launch_router_logits(const uint16_t* x, const float* w, int T, int H, int E, float* logits,
                                 cudaStream_t s) {
  if (T <= kMaxSmallRouterTokens) {
    router_gemv_kernel<<<E, 256, 0, s>>>(x, w, T, H, E, logits);
    return cudaGetLastError();
  }
  const int splits = router_split_count(T, H, E);
  dim3 grid((E + RBN - 1) / RBN, (T + RBM - 1) / RBM, splits);
  return launch_pdl(router_sgemm_kernel, grid, dim3(256), 0, s, x, w, T, H, E, H / splits, logits);
}

// ------------------------------------------------------------------ top-k
template <int EPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ partial, int splits, int T, int E, int k,
                                                   int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  // slices outer, experts inner: the EPL loads of one slice are in flight together (the
  // partials are read once: streaming loads); each expert's sum still runs over the slices
  // in order
  float v[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) v[i] = lane + 32 * i < E ? 0.0f : -INFINITY;
  for (int sp = 0; sp < splits; ++sp) {
    const float* row = partial + (static_cast<size_t>(sp) * T + t) * E;
    float p[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) p[i] = lane + 32 * i < E ? __ldcs(row + lane + 32 * i) : 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] += p[i];
  }
  warp_topk<EPL>(v, E, k, lane, ids + static_cast<size_t>(t) * k, wout + static_cast<size_t>(t) * k);
}

cudaError_t launch_topk(const float* logits, int splits, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t s) {
  const int blocks = (T + 7) / 8;
  const int epl = (E + 31) / 32;
  if (epl <= 1) return launch_pdl(topk_kernel<1>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
  if (epl <= 2) return launch_pdl(topk_kernel<2>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
  if (epl <= 4) return launch_pdl(topk_kernel<4>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
  if (epl <= 8) return launch_pdl(topk_kernel<8>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
  if (epl <= 16) return launch_pdl(topk_kernel<16>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
  return launch_pdl(topk_kernel<32>, dim3(blocks), dim3(256), 0, s, logits, splits, T, E, k, ids, w);
}

}  // namespace beam
