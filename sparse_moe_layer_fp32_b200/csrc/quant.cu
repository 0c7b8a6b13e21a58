// NVFP4 quantiser for whole tensors (weights at load time, or any FP32 tensor) and the
// create-time repacking of expert weights into the tensor-core operand layout.
//
// NVFP4 (recipe "reflection/Beam-1.0-501B-A23B", section "Variants": NVFP4 routed
// experts, W4A4 on Blackwell): E2M1 codes, one unsigned E4M3 scale per 16 values of a
// row, one FP32 tensor scale alpha = amax / 2688 per tensor.  Every step is an IEEE FP32
// operation with round-to-nearest-even (division by __fdiv_rn, conversions by
// cvt.rn.satfinite), so the codes do not depend on the launch shape.
//
// MXFP8, the block-scaled FP8 variant of the experts (the recipe's FP8 checkpoint, same
// section; read as the OCP microscaling format): E4M3 codes, one UE8M0 power-of-two scale
// per 32 values of a row, no tensor scale.  Its quantiser and weight repack are at the end.
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
// Returns the source row (rows 0..I-1 gate, I..2I-1 up) of interleaved row lr.
__device__ __forceinline__ int gate_up_src_row(int lr, int I) {
  const int fb = lr >> 8, g = (lr >> 7) & 1, i = lr & 127;
  return g * I + fb * 128 + i;
}

// Weights as contiguous B tiles for the grouped GEMMs.  Tile (e, nt, kt) covers rows
// [256 nt, 256 nt + 256) of expert e (after the gate/up interleave) and K values
// [256 kt, 256 kt + 256): kTileCodeBytes of codes laid out exactly as the tensor core
// reads them from shared memory (row r at r * 128, 16-byte chunk c of the row at
// ((c ^ (r % 8)) * 16): the 128-byte swizzle), then kTileSfBytes of scales (two 128-row
// blocks, each 4 K-groups x 512 bytes in the tcgen05 scale-factor layout).  One bulk copy
// moves a whole tile.
__global__ void repack_tiles_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int E,
                                    int rows_per_e, int K, int Kp, int interleave_inter, uint8_t* __restrict__ dst) {
  const int n_tiles = rows_per_e / 256, k_tiles = Kp / 256;
  constexpr int kChunks = kTileBytes / 16;  // 16-byte chunks per tile
  const int64_t total = static_cast<int64_t>(E) * n_tiles * k_tiles * kChunks;
  const int src_row_bytes = K / 2, src_scales = K / 16;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = q / kChunks;
    const int o = static_cast<int>(q % kChunks) * 16;  // byte offset in the tile
    const int kt = static_cast<int>(tile % k_tiles);
    const int nt = static_cast<int>((tile / k_tiles) % n_tiles);
    const int e = static_cast<int>(tile / (static_cast<int64_t>(k_tiles) * n_tiles));
    uint4 v = make_uint4(0, 0, 0, 0);
    if (o < kTileCodeBytes) {
      // shared-memory slot (o >> 4) & 7 of row r holds logical 16-byte chunk slot ^ (r % 8)
      const int r = o >> 7, c = ((o >> 4) & 7) ^ (r & 7);
      const int lr = nt * 256 + r;
      const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
      const int byte = kt * 128 + c * 16;  // K/2 is a multiple of 64: a chunk is all in or all out
      if (byte < src_row_bytes)
        v = *reinterpret_cast<const uint4*>(codes + (static_cast<int64_t>(e) * rows_per_e + slr) * src_row_bytes + byte);
    } else {
      uint8_t b[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int so = o - kTileCodeBytes + i;
        const int nb = so >> 11, kb = (so >> 9) & 3, a = so & 511;
        const int m = (a >> 4) + 32 * ((a & 15) >> 2);
        const int sidx = (kt * 4 + kb) * 4 + (a & 3);
        const int lr = nt * 256 + nb * 128 + m;
        const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
        b[i] = sidx < src_scales ? sf[(static_cast<int64_t>(e) * rows_per_e + slr) * src_scales + sidx] : 0;
      }
      v.x = b[0] | (b[1] << 8) | (b[2] << 16) | (static_cast<uint32_t>(b[3]) << 24);
      v.y = b[4] | (b[5] << 8) | (b[6] << 16) | (static_cast<uint32_t>(b[7]) << 24);
      v.z = b[8] | (b[9] << 8) | (b[10] << 16) | (static_cast<uint32_t>(b[11]) << 24);
      v.w = b[12] | (b[13] << 8) | (b[14] << 16) | (static_cast<uint32_t>(b[15]) << 24);
    }
    *reinterpret_cast<uint4*>(dst + tile * kTileBytes + o) = v;
  }
}

static int grid_for(int64_t work) {
  const int64_t want = (work + 255) / 256;
  return static_cast<int>(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
}

cudaError_t launch_repack_tiles(const uint8_t* codes, const uint8_t* sf, int E, int rows_per_e, int K, int Kp,
                                int interleave_inter, uint8_t* dst, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(E) * (rows_per_e / 256) * (Kp / 256) * (kTileBytes / 16);
  repack_tiles_kernel<<<grid_for(total), 256, 0, s>>>(codes, sf, E, rows_per_e, K, Kp, interleave_inter, dst);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ MXFP8
// MXFP8 (block-scaled FP8 experts, E4M3 + one UE8M0 scale per 32 values): one thread per
// 32-value block of a row-major tensor whose rows hold whole blocks.  The rule is exact
// (quant_block32_mx), so the codes do not depend on the launch shape.
__global__ void __launch_bounds__(256) quantize_blocks_mx_kernel(const float* __restrict__ src, int64_t nblocks,
                                                                 uint8_t* __restrict__ codes,
                                                                 uint8_t* __restrict__ sf) {
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < nblocks;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4* p = reinterpret_cast<const float4*>(src + q * 32);
    float v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 f = __ldg(p + i);
      v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
    }
    uint32_t c[8];
    const uint32_t sc = quant_block32_mx(v, c);
    uint4* d = reinterpret_cast<uint4*>(codes + q * 32);
    d[0] = make_uint4(c[0], c[1], c[2], c[3]);
    d[1] = make_uint4(c[4], c[5], c[6], c[7]);
    sf[q] = static_cast<uint8_t>(sc);
  }
}

cudaError_t launch_quantize_rows_mx(const float* src, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* sf,
                                    cudaStream_t s) {
  const int64_t nblocks = rows * (cols / 32);
  if (nblocks == 0) return cudaSuccess;
  const int64_t want = (nblocks + 255) / 256;
  const int grid = static_cast<int>(want < 148 * 16 ? want : 148 * 16);
  quantize_blocks_mx_kernel<<<grid, 256, 0, s>>>(src, nblocks, codes, sf);
  return cudaGetLastError();
}

// MXFP8 weight tiles.  Tile (e, nt, kt) covers rows [256 nt, 256 nt + 256) of expert e (after
// the gate/up interleave) and K values [128 kt, 128 kt + 128): kTileCodeBytes of E4M3 codes
// in the 128-byte swizzle (row r at r * 128, chunk c at ((c ^ (r % 8)) * 16)), then two
// 512-byte scale atoms (rows 0-127, rows 128-255).  Atom byte a holds the scale of row
// (a / 16) + 32 ((a % 16) / 4) for the 32-value block (a % 4) of the tile's K range, so
// each 32-bit word is the 4 scales of one row and TMEM lane m finds row m's word in
// column m / 32.
__global__ void repack_tiles_mx_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sf, int E,
                                       int rows_per_e, int K, int interleave_inter, uint8_t* __restrict__ dst) {
  const int n_tiles = rows_per_e / 256, k_tiles = K / 128;
  constexpr int kChunks = kMxTileBytes / 16;
  const int64_t total = static_cast<int64_t>(E) * n_tiles * k_tiles * kChunks;
  const int src_scales = K / 32;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t tile = q / kChunks;
    const int o = static_cast<int>(q % kChunks) * 16;
    const int kt = static_cast<int>(tile % k_tiles);
    const int nt = static_cast<int>((tile / k_tiles) % n_tiles);
    const int e = static_cast<int>(tile / (static_cast<int64_t>(k_tiles) * n_tiles));
    uint4 v;
    if (o < kTileCodeBytes) {
      const int r = o >> 7, c = ((o >> 4) & 7) ^ (r & 7);
      const int lr = nt * 256 + r;
      const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
      v = *reinterpret_cast<const uint4*>(codes + (static_cast<int64_t>(e) * rows_per_e + slr) * K + kt * 128 +
                                          c * 16);
    } else {
      uint8_t b[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int so = o - kTileCodeBytes + i;
        const int nb = so >> 9, a = so & 511;
        const int m = (a >> 4) + 32 * ((a & 15) >> 2);
        const int lr = nt * 256 + nb * 128 + m;
        const int slr = interleave_inter ? gate_up_src_row(lr, interleave_inter) : lr;
        b[i] = sf[(static_cast<int64_t>(e) * rows_per_e + slr) * src_scales + kt * 4 + (a & 3)];
      }
      v.x = b[0] | (b[1] << 8) | (b[2] << 16) | (static_cast<uint32_t>(b[3]) << 24);
      v.y = b[4] | (b[5] << 8) | (b[6] << 16) | (static_cast<uint32_t>(b[7]) << 24);
      v.z = b[8] | (b[9] << 8) | (b[10] << 16) | (static_cast<uint32_t>(b[11]) << 24);
      v.w = b[12] | (b[13] << 8) | (b[14] << 16) | (static_cast<uint32_t>(b[15]) << 24);
    }
    *reinterpret_cast<uint4*>(dst + tile * kMxTileBytes + o) = v;
  }
}

cudaError_t launch_repack_tiles_mx(const uint8_t* codes, const uint8_t* sf, int E, int rows_per_e, int K,
                                   int interleave_inter, uint8_t* dst, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(E) * (rows_per_e / 256) * (K / 128) * (kMxTileBytes / 16);
  repack_tiles_mx_kernel<<<grid_for(total), 256, 0, s>>>(codes, sf, E, rows_per_e, K, interleave_inter, dst);
  return cudaGetLastError();
}

}  // namespace beam
