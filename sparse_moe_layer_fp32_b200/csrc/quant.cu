// NVFP4 quantiser for whole tensors (weights at load time, or any FP32 tensor) and the
// create-time repacking of expert weights into the tensor-core operand layout.
//
// NVFP4 (recipe "reflection/Beam-1.0-501B-A23B", section "Variants": NVFP4 routed
// experts, W4A4 on Blackwell): E2M1 codes, one unsigned E4M3 scale per 16 values of a
// row, one FP32 tensor scale alpha = amax / 2688 per tensor.  Every step is an IEEE FP32
// operation with round-to-nearest-even (division by __fdiv_rn, conversions by
// cvt.rn.satfinite), so the codes do not depend on the launch shape.
#include "common.cuh"
#include "internal.h"

namespace beam {

// One thread per 16-value block of a row-major tensor whose rows hold whole blocks.
__global__ void __launch_bounds__(256) quantize_blocks_kernel(const float* __restrict__ src, int64_t nblocks,
                                                              float alpha_param,
                                                              const float* __restrict__ amax_dev,
                                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const float alpha = amax_dev ? __fdiv_rn(*amax_dev, 2688.0f) : alpha_param;
  const float six_alpha = __fmul_rn(6.0f, alpha);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < nblocks;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4* p = reinterpret_cast<const float4*>(src + q * 16);
    float v[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 f = __ldg(p + i);
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    uint32_t lo = 0, hi = 0, sc = 0;
    if (alpha > 0.0f) sc = quant_block16(v, alpha, six_alpha, lo, hi);
    *reinterpret_cast<uint2*>(codes + q * 8) = make_uint2(lo, hi);
    sf[q] = static_cast<uint8_t>(sc);
  }
}

// amax of |src| as FP32 bits; non-negative floats order like their bit patterns.
__global__ void __launch_bounds__(256) amax_kernel(const float* __restrict__ src, int64_t n,
                                                   unsigned int* __restrict__ out) {
  float m = 0.0f;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    m = fmaxf(m, fabsf(src[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < 8; ++i) m = fmaxf(m, wm[i]);
    atomicMax(out, __float_as_uint(m));
  }
}

__global__ void amax_to_alpha_kernel(float* p) { *p = __fdiv_rn(*p, 2688.0f); }

cudaError_t launch_amax(const float* src, int64_t n, float* amax_bits, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(amax_bits, 0, sizeof(float), s);
  if (e != cudaSuccess) return e;
  const int64_t want = (n + 255) / 256;
  const int grid = static_cast<int>(want < 148 * 8 ? (want > 0 ? want : 1) : 148 * 8);
  amax_kernel<<<grid, 256, 0, s>>>(src, n, reinterpret_cast<unsigned int*>(amax_bits));
  return cudaGetLastError();
}

cudaError_t launch_amax_to_alpha(float* inout, cudaStream_t s) {
  amax_to_alpha_kernel<<<1, 1, 0, s>>>(inout);
  return cudaGetLastError();
}

cudaError_t launch_quantize_rows(const float* src, int64_t rows, int64_t cols, float alpha, const float* amax_dev,
                                 uint8_t* codes, uint8_t* sf, cudaStream_t s) {
  const int64_t nblocks = rows * (cols / 16);
  if (nblocks == 0) return cudaSuccess;
  const int64_t want = (nblocks + 255) / 256;
  const int grid = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  quantize_blocks_kernel<<<grid, 256, 0, s>>>(src, nblocks, alpha, amax_dev, codes, sf);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ repacking
// Gate/up rows are interleaved per 128-feature block b: rows [256b, 256b+128) are gate
// features [128b, 128b+128) and rows [256b+128, 256b+256) the matching up features, so
// one 256-row B tile gives an epilogue thread both halves of SwiGLU for 128 features.
__device__ __forceinline__ int gate_up_src_row(int lr, int I) {
  const int fb = lr >> 8, g = (lr >> 7) & 1, i = lr & 127;
  return g * I + fb * 128 + i;
}

__global__ void repack_rows_kernel(const uint8_t* __restrict__ src, int E, int rows_per_e, int src_bytes,
                                   int dst_bytes, int interleave_inter, uint8_t* __restrict__ dst) {
  // one thread per 16 bytes of destination
  const int64_t chunks_per_row = dst_bytes / 16;
  const int64_t total = static_cast<int64_t>(E) * rows_per_e * chunks_per_row;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = q / chunks_per_row;
    const int c = static_cast<int>(q % chunks_per_row);
    const int e = static_cast<int>(row / rows_per_e), lr = static_cast<int>(row % rows_per_e);
    const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (c * 16 < src_bytes)
      v = *reinterpret_cast<const uint4*>(src + (static_cast<int64_t>(e) * rows_per_e + slr) * src_bytes + c * 16);
    *reinterpret_cast<uint4*>(dst + row * dst_bytes + c * 16) = v;
  }
}

// Scale bytes [E][rows][src_scales] -> 128-row scale blocks [E][rows/128][kgroups][512].
__global__ void repack_sf_kernel(const uint8_t* __restrict__ src, int E, int rows_per_e, int src_scales,
                                 int kgroups, int interleave_inter, uint8_t* __restrict__ dst) {
  const int64_t total = static_cast<int64_t>(E) * (rows_per_e / 128) * kgroups * 512;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(q & 511);
    const int64_t blk_k = q >> 9;
    const int kg = static_cast<int>(blk_k % kgroups);
    const int64_t blk = blk_k / kgroups;  // global block index = e * (rows/128) + rb
    const int e = static_cast<int>(blk / (rows_per_e / 128)), rb = static_cast<int>(blk % (rows_per_e / 128));
    const int m = (o >> 4) + 32 * ((o & 15) >> 2);
    const int sidx = kg * 4 + (o & 3);
    const int lr = rb * 128 + m;
    const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
    uint8_t v = 0;
    if (sidx < src_scales) v = src[(static_cast<int64_t>(e) * rows_per_e + slr) * src_scales + sidx];
    dst[q] = v;
  }
}

static int grid_for(int64_t work) {
  const int64_t want = (work + 255) / 256;
  return static_cast<int>(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
}

cudaError_t launch_repack_gate_up(const uint8_t* codes, const uint8_t* sf, int E, int I, int H, uint8_t* codes_out,
                                  uint8_t* sf_out, cudaStream_t s) {
  const int rows = 2 * I;
  repack_rows_kernel<<<grid_for(static_cast<int64_t>(E) * rows * (H / 32)), 256, 0, s>>>(codes, E, rows, H / 2,
                                                                                        H / 2, I, codes_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  repack_sf_kernel<<<grid_for(static_cast<int64_t>(E) * rows * (H / 16)), 256, 0, s>>>(sf, E, rows, H / 16, H / 64,
                                                                                      I, sf_out);
  return cudaGetLastError();
}

cudaError_t launch_repack_down(const uint8_t* codes, const uint8_t* sf, int E, int I, int Ip, int H,
                               uint8_t* codes_out, uint8_t* sf_out, cudaStream_t s) {
  repack_rows_kernel<<<grid_for(static_cast<int64_t>(E) * H * (Ip / 32)), 256, 0, s>>>(codes, E, H, I / 2, Ip / 2,
                                                                                      0, codes_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  repack_sf_kernel<<<grid_for(static_cast<int64_t>(E) * H * (Ip / 16)), 256, 0, s>>>(sf, E, H, I / 16, Ip / 64, 0,
                                                                                    sf_out);
  return cudaGetLastError();
}

}  // namespace beam
