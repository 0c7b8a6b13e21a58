// Routing of a small batch (T <= 16 tokens, E <= 256 experts) in one launch: router
// logits, top-k + renormalise, histogram, scan, permutation and the 128-row work blocks.
//
// Phase 1 (every CTA): each CTA streams the rows W_r[e] of 4 experts (20 KB each at
// H = 5120) into registers, stages x (T x H BF16) once in shared memory, and dots every
// token with the 4 rows in FP32.  All loads are issued before any multiply; the step is
// bound by reading W_r.
// Phase 2 (the last CTA to finish, found with an atomic counter after a release fence):
// top-k per token (one warp per token), then the histogram, the prefix sums and the
// stable permutation for the whole batch, as routing.cu does in three launches for large
// batches.  The counter is reset by that CTA, ready for the next launch.
// Router (5120 -> 256 experts, FP32): vLLM PR "Day-0 support for Reflection's Beam-1.0",
// section "Status"; news article "vLLM adds day-zero Reflection Beam serving", section
// "Agents worked on the serving path".  8 of 256 experts: recipe
// "reflection/Beam-1.0-501B-A23B", section "Overview".
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace beam {

constexpr int kSmallThreads = 256;
constexpr int kExpertsPerCta = 4;       // x is staged once per CTA and reused for 4 experts
constexpr int kMaxChunksPerThread = 8;  // H / 4 / 256 <= 8  ->  H <= 8192

__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E, int k,
    float* __restrict__ logits, int32_t* __restrict__ ids, float* __restrict__ wout, int32_t* __restrict__ offsets,
    int32_t* __restrict__ sf_block, MBlock* __restrict__ mblocks, int32_t* __restrict__ num_mblocks,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, unsigned int* __restrict__ done_counter) {
  extern __shared__ __align__(16) uint16_t xs[];  // [T][H] BF16
  const int e0 = blockIdx.x * kExpertsPerCta;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n4 = H / 4;
  // ---------------------------------------------------------------- phase 1: logits
  {
    // The router weights are constant: stream this CTA's rows before waiting for the
    // previous kernel in the stream.
    float4 wv[kExpertsPerCta][kMaxChunksPerThread];
#pragma unroll
    for (int q = 0; q < kExpertsPerCta; ++q) {
      const float4* wr = reinterpret_cast<const float4*>(w + static_cast<size_t>(min(e0 + q, E - 1)) * H);
#pragma unroll
      for (int i = 0; i < kMaxChunksPerThread; ++i) {
        const int c = tid + i * kSmallThreads;
        wv[q][i] = (c < n4 && e0 + q < E) ? __ldg(wr + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    pdl_wait();
    pdl_trigger();
    {  // x -> shared memory: asynchronous 16-byte copies, all in flight at once
      const int n16 = T * H / 8;
      const uint4* xg = reinterpret_cast<const uint4*>(x);
      for (int i = tid; i < n16; i += kSmallThreads)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(xs + 8 * i)), "l"(xg + i) : "memory");
      asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    __shared__ float part[kSmallThreads / 32][kExpertsPerCta][kMaxSmallRouterTokens];
    for (int t = 0; t < T; ++t) {
      const uint2* xr = reinterpret_cast<const uint2*>(xs + static_cast<size_t>(t) * H);
      float acc[kExpertsPerCta] = {};
#pragma unroll
      for (int i = 0; i < kMaxChunksPerThread; ++i) {
        const int c = tid + i * kSmallThreads;
        if (c < n4) {
          const uint2 xv = xr[c];
          const float x0 = bf16_bits_to_f32(xv.x & 0xFFFFu), x1 = bf16_bits_to_f32(xv.x >> 16);
          const float x2 = bf16_bits_to_f32(xv.y & 0xFFFFu), x3 = bf16_bits_to_f32(xv.y >> 16);
#pragma unroll
          for (int q = 0; q < kExpertsPerCta; ++q) {
            acc[q] = fmaf(x0, wv[q][i].x, acc[q]);
            acc[q] = fmaf(x1, wv[q][i].y, acc[q]);
            acc[q] = fmaf(x2, wv[q][i].z, acc[q]);
            acc[q] = fmaf(x3, wv[q][i].w, acc[q]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kExpertsPerCta; ++q) {
        float a = acc[q];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (lane == 0) part[warp][q][t] = a;
      }
    }
    __syncthreads();
    for (int i = tid; i < kExpertsPerCta * T; i += kSmallThreads) {
      const int q = i / T, t = i % T;
      if (e0 + q >= E) continue;
      float v = 0.0f;
#pragma unroll
      for (int g = 0; g < kSmallThreads / 32; ++g) v += part[g][q][t];
      logits[static_cast<size_t>(t) * E + e0 + q] = v;
    }
  }
  // ---------------------------------------------------------------- elect the last CTA
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(done_counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---------------------------------------------------------------- phase 2: top-k
  __shared__ int s_ids[kMaxSmallRouterTokens * 16];
  __shared__ int s_cnt[256];
  __shared__ int s_off[256];
  __shared__ int warp_sums[33];
  for (int t = warp; t < T; t += kSmallThreads / 32) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      v[i] = ee < E ? __ldcg(logits + static_cast<size_t>(t) * E + ee) : -INFINITY;
    }
    warp_topk<8>(v, E, k, lane, ids + static_cast<size_t>(t) * k, wout + static_cast<size_t>(t) * k);
  }
  __syncthreads();  // ids of this CTA's writes are visible to the CTA after the barrier
  const int R = T * k;
  for (int i = tid; i < R; i += kSmallThreads) s_ids[i] = ids[i];
  for (int i = tid; i < E; i += kSmallThreads) s_cnt[i] = 0;
  __syncthreads();
  for (int i = tid; i < R; i += kSmallThreads) atomicAdd(&s_cnt[s_ids[i]], 1);
  __syncthreads();
  // ---------------------------------------------------------------- scan and work blocks
  const int cnt = tid < E ? s_cnt[tid] : 0;
  const int nblk = (cnt + 127) / 128;
  int total_rows, total_blk;
  const int off = block_exclusive_scan(cnt, warp_sums, total_rows);
  const int blk = block_exclusive_scan(nblk, warp_sums, total_blk);
  if (tid < E) {
    offsets[tid] = off;
    sf_block[tid] = blk;
    s_off[tid] = off;
    for (int i = 0; i < nblk; ++i) {
      MBlock m;
      m.expert = tid;
      m.row_begin = off + 128 * i;
      m.rows = min(128, cnt - 128 * i);
      m.sf_block = blk + i;
      mblocks[blk + i] = m;
    }
  }
  if (tid == 0) {
    offsets[E] = total_rows;
    sf_block[E] = total_blk;
    *num_mblocks = total_blk;
  }
  __syncthreads();
  // ---------------------------------------------------------------- permutation
  // rank of (t, j) = number of earlier tokens that chose the same expert
  for (int i = tid; i < R; i += kSmallThreads) {
    const int t = i / k, ee = s_ids[i];
    int rank = 0;
    for (int q = 0; q < t * k; ++q) rank += s_ids[q] == ee;
    const int r = s_off[ee] + rank;
    perm[r] = t;
    inv[i] = r;
  }
  if (tid == 0) *done_counter = 0u;
}

bool route_small_supported(int T, int H, int E, int k) {
  return T >= 1 && T <= kMaxSmallRouterTokens && E <= 256 && k <= 16 && H / 4 <= kMaxChunksPerThread * kSmallThreads &&
         static_cast<size_t>(T) * H * 2 <= 160 * 1024;
}

cudaError_t launch_route_small(const uint16_t* x, const float* w, int T, int H, int E, int k, float* logits,
                               int32_t* ids, float* wout, int32_t* offsets, int32_t* sf_block, MBlock* mblocks,
                               int32_t* num_mblocks, int32_t* perm, int32_t* inv, unsigned int* done_counter,
                               cudaStream_t s) {
  const size_t smem = static_cast<size_t>(T) * H * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(route_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(route_small_kernel, dim3((E + kExpertsPerCta - 1) / kExpertsPerCta), dim3(kSmallThreads), smem,
                    s, x, w, T, H, E, k, logits, ids, wout, offsets, sf_block, mblocks, num_mblocks, perm, inv,
                    done_counter);
}

}  // namespace beam
