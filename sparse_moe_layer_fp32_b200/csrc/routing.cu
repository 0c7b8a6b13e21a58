// Token -> expert histogram, prefix scan, permutation, and the NVFP4 quantisation of the
// expert inputs fused into the permute.
//
// The permuted order lists the (token, slot) pairs of expert e in rows
// [offsets[e], offsets[e+1]), in ascending token order.  It is deterministic: the rank
// of token t among the tokens of its chunk that chose expert e is a popcount of a
// per-warp bitmask (OR is order-independent), and chunk bases come from a sequential
// per-expert scan over chunks.  Each expert's rows are also cut into 128-row work blocks
// (the M tiles of the grouped GEMMs), each with its own scale block so the tensor-core
// scale layout stays aligned to 128 rows whatever offsets[e] is.
//
// A1 = Q(x, alpha_a1): x rows are quantised once per token (16-value blocks along H) and
// the codes are written to the token's k permuted rows (the NVFP4 W4A4 experts of the
// recipe "reflection/Beam-1.0-501B-A23B", section "Variants"), as activation tiles (see
// act_tile_offset) of the row's 128-row block, each K step's scales after its codes
// (sf_chunk_offset).  For the block-scaled FP8 variant of the experts (the recipe's FP8
// checkpoint, read as MXFP8), A1 = MX(x) in 32-value blocks.
#include "common.cuh"
#include "internal.h"

namespace beam {

// chunk_counts[c][e] = number of (t, j) in chunk c with ids[t][j] == e
__global__ void __launch_bounds__(256) chunk_hist_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                         int32_t* __restrict__ chunk_counts) {
  extern __shared__ int32_t cnt[];
  pdl_wait();
  pdl_trigger();
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kChunkTokens;
  const int n = min(kChunkTokens, T - t0) * k;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = ids[static_cast<size_t>(t0) * k + i];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_counts[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

// One CTA, one thread per expert.
__global__ void scan_kernel(const int32_t* __restrict__ chunk_counts, int n_chunks, int E,
                            int32_t* __restrict__ chunk_base, int32_t* __restrict__ offsets,
                            int32_t* __restrict__ sf_block, MBlock* __restrict__ mblocks,
                            int32_t* __restrict__ num_mblocks, uint32_t* __restrict__ sched, int sched_n,
                            BlockScales bs) {
  __shared__ int warp_sums[33];
  pdl_wait();
  pdl_trigger();
  // the expert GEMM launch that follows starts from zeroed scheduler words
  for (int i = threadIdx.x; i < sched_n; i += blockDim.x) sched[i] = 0u;
  const int e = threadIdx.x;
  int cnt = 0;
  if (e < E) {
    for (int c = 0; c < n_chunks; ++c) {
      const size_t i = static_cast<size_t>(c) * E + e;
      const int v = chunk_counts[i];
      chunk_base[i] = cnt;
      cnt += v;
    }
  }
  // Activations live in 128-row blocks (sf_block), and so does the work list.
  const int nblk = (cnt + 127) / 128;
  const bool held = e >= bs.e_begin && e < bs.e_end;  // this handle has the expert's weights
  const int nwork = held ? nblk : 0;
  int total_rows, total_blk, total_work;
  const int off = block_exclusive_scan(cnt, warp_sums, total_rows);
  const int blk = block_exclusive_scan(nblk, warp_sums, total_blk);
  const int wbase = block_exclusive_scan(nwork, warp_sums, total_work);
  if (e < E) {
    offsets[e] = off;
    sf_block[e] = blk;
    for (int c = 0; c < n_chunks; ++c) chunk_base[static_cast<size_t>(c) * E + e] += off;
    for (int i = 0; i < nwork; ++i) {
      MBlock m;
      m.expert = e - bs.e_begin;
      m.row_begin = off + 128 * i;
      m.rows = min(128, cnt - 128 * i);
      m.sf_block = blk + i;
      m.scale_gu = bs.alpha_a1 * __ldg(bs.w_gu_alpha + m.expert);
      m.scale_d = bs.alpha_a2 * __ldg(bs.w_d_alpha + m.expert);
      m.pad[0] = m.pad[1] = 0;
      mblocks[wbase + i] = m;
    }
  }
  if (e == 0) {
    offsets[E] = total_rows;
    sf_block[E] = total_blk;
    *num_mblocks = total_work;
  }
}

// perm_src[r] = t, inv[t][j] = r and tile_row[t][j] (128 x activation block + row in the
// block, the row's place in the activation tiles) for every (t, j) of one chunk of 256
// tokens.
__global__ void __launch_bounds__(256) scatter_kernel(const int32_t* __restrict__ ids,
                                                      const int32_t* __restrict__ chunk_base,
                                                      const int32_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ sf_block, int T, int k, int E,
                                                      int32_t* __restrict__ perm_src, int32_t* __restrict__ inv,
                                                      int32_t* __restrict__ tile_row) {
  extern __shared__ uint32_t sm[];
  uint32_t* mask = sm;                                    // [8][E]
  int32_t* pre = reinterpret_cast<int32_t*>(sm + 8 * E);  // [8][E]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) mask[i] = 0;
  __syncthreads();
  const int chunk = blockIdx.x;
  const int t = chunk * kChunkTokens + warp * 32 + lane;
  if (t < T)
    for (int j = 0; j < k; ++j) atomicOr(&mask[warp * E + ids[static_cast<size_t>(t) * k + j]], 1u << lane);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      pre[w * E + e] = run;
      run += __popc(mask[w * E + e]);
    }
  }
  __syncthreads();
  if (t < T) {
    const uint32_t below = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = ids[static_cast<size_t>(t) * k + j];
      const int rank = pre[warp * E + e] + __popc(mask[warp * E + e] & below);
      const int r = chunk_base[static_cast<size_t>(chunk) * E + e] + rank;
      const int li = r - offsets[e];  // row within the expert
      perm_src[r] = t;
      inv[static_cast<size_t>(t) * k + j] = r;
      tile_row[static_cast<size_t>(t) * k + j] = (sf_block[e] + (li >> 7)) * 128 + (li & 127);
    }
  }
}

// One thread per 16-value block of x: quantise it once and write it to the token's k
// permuted rows.  The four threads of one 64-value group (one scale word of the
// tensor-core layout) combine their scale bytes and one of them stores the 32-bit word.
__global__ void __launch_bounds__(128) quant_a1_kernel(const uint16_t* __restrict__ x,
                                                       const int32_t* __restrict__ tile_row, int T, int H, int k,
                                                       float alpha, uint8_t* __restrict__ a1) {
  const int nb = H / 16;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool active = gid < static_cast<int64_t>(T) * nb;
  const int t = active ? static_cast<int>(gid / nb) : 0;
  const int b = active ? static_cast<int>(gid % nb) : 0;
  pdl_wait();
  pdl_trigger();
  uint32_t lo = 0, hi = 0, sc = 0;
  int dst[16];
  if (active) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
    const uint4 p0 = __ldg(xr + 2 * b), p1 = __ldg(xr + 2 * b + 1);
#pragma unroll
    for (int j = 0; j < 16; ++j)  // all slot rows in flight together
      dst[j] = j < k ? __ldg(tile_row + static_cast<size_t>(t) * k + j) : 0;
    const uint32_t u[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    float v[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
    }
    sc = quant_block16(v, alpha, __fmul_rn(6.0f, alpha), lo, hi);
  }
  // lanes 4q..4q+3 hold blocks 4g..4g+3 of one token (nb is a multiple of 4)
  const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
  const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
  const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
  const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
  if (!active) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j >= k) break;
    const int blk = dst[j] >> 7, m = dst[j] & 127;
    // block b of 16 values: 8 bytes, half of 16-byte chunk (b % 16) / 2 of K tile b / 16
    *reinterpret_cast<uint2*>(a1 + act_tile_offset(blk, H / 256, b >> 4, m, (b & 15) >> 1) + (b & 1) * 8) =
        make_uint2(lo, hi);
    if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(a1 + sf_chunk_offset(blk, H / 256, m, b)) = word;
  }
}

// Large batches: one warp per token, quantise x[t] once, write it to the token's k rows.
__global__ void __launch_bounds__(256) quant_a1_wide_kernel(const uint16_t* __restrict__ x,
                                                       const int32_t* __restrict__ tile_row, int T, int H,
                                                       int k, float alpha, uint8_t* __restrict__ a1) {
  __shared__ int s_blk[8][16], s_m[8][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  // lane j < k: the permuted row of slot j and where its scales live
  if (lane < k) {
    const int d = tile_row[static_cast<size_t>(t) * k + lane];
    s_blk[warp][lane] = d >> 7;
    s_m[warp][lane] = d & 127;
  }
  __syncwarp();
  const float six_alpha = __fmul_rn(6.0f, alpha);
  const int nb = H / 16;
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  // Lanes 2c, 2c + 1 hold the two halves of one 16-byte code chunk and lanes 4g..4g + 3 the
  // four scale bytes of one K-group (nb is a multiple of 4): one 16-byte code store per lane
  // pair and one 4-byte scale store per lane quad, per slot.  The next iteration's 32 bytes
  // are loaded before this one's quantisation (its divisions hide the load latency).
  uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
  if (lane < nb) {
    n0 = __ldg(xr + 2 * lane);
    n1 = __ldg(xr + 2 * lane + 1);
  }
  for (int b0 = 0; b0 < nb; b0 += 32) {
    const int b = b0 + lane;
    const bool active = b < nb;  // whole quads are active or not
    const uint4 p0 = n0, p1 = n1;
    if (b + 32 < nb) {
      n0 = __ldg(xr + 2 * (b + 32));
      n1 = __ldg(xr + 2 * (b + 32) + 1);
    }
    uint32_t lo = 0, hi = 0, sc = 0;
    if (active) {
      const uint32_t u[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      float v[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
      }
      sc = quant_block16(v, alpha, six_alpha, lo, hi);
    }
    const uint32_t lo1 = __shfl_down_sync(0xffffffffu, lo, 1), hi1 = __shfl_down_sync(0xffffffffu, hi, 1);
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
    const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
    if (!active || (lane & 1)) continue;
    for (int j = 0; j < k; ++j) {
      const int blk = s_blk[warp][j], m = s_m[warp][j];
      *reinterpret_cast<uint4*>(a1 + act_tile_offset(blk, H / 256, b >> 4, m, (b & 15) >> 1)) =
          make_uint4(lo, hi, lo1, hi1);
      if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(a1 + sf_chunk_offset(blk, H / 256, m, b)) = word;
    }
  }
}

// ------------------------------------------------------------------ MXFP8
// A1 = MX(x) for MXFP8 experts (E4M3 codes, one UE8M0 scale per 32 values): one thread per
// 32-value block of x, quantised once and written to the token's k permuted rows.  A
// block's 32 codes are chunks 2 (b % 4) and 2 (b % 4) + 1 of K tile b / 4 (one 32-byte
// store); the four threads of one K tile combine their scale bytes into the row's 32-bit
// scale word of that tile and one of them stores it.
__device__ __forceinline__ void load_block32_bf16(const uint16_t* __restrict__ x, size_t t, int H, int b,
                                                  float (&v)[32]) {
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * H) + 4 * b;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 p = __ldg(xr + q);
    const uint32_t u[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
      v[8 * q + 2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
    }
  }
}

__global__ void __launch_bounds__(128) quant_a1_mx_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ tile_row, int T, int H, int k,
                                                          uint8_t* __restrict__ a1) {
  const int nb = H / 32, k_tiles = H / 128;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool active = gid < static_cast<int64_t>(T) * nb;
  const int t = active ? static_cast<int>(gid / nb) : 0;
  const int b = active ? static_cast<int>(gid % nb) : 0;
  pdl_wait();
  pdl_trigger();
  uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sc = 0;
  int dst[16];
  if (active) {
#pragma unroll
    for (int j = 0; j < 16; ++j) dst[j] = j < k ? __ldg(tile_row + static_cast<size_t>(t) * k + j) : 0;
    float v[32];
    load_block32_bf16(x, t, H, b, v);
    sc = quant_block32_mx(v, c);
  }
  // lanes 4q..4q+3 hold blocks 4g..4g+3 of one token (nb is a multiple of 8)
  const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
  const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
  const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
  const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
  if (!active) return;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j >= k) break;
    const int blk = dst[j] >> 7, m = dst[j] & 127;
    st_act_pair(a1, blk, k_tiles, b >> 2, m, (b & 3) * 2, c);
    if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(a1 + sf_atom_offset(blk, k_tiles, m, b)) = word;
  }
}

// Large batches: one warp per token, lane = 32-value block.
__global__ void __launch_bounds__(256) quant_a1_mx_wide_kernel(const uint16_t* __restrict__ x,
                                                               const int32_t* __restrict__ tile_row, int T, int H,
                                                               int k, uint8_t* __restrict__ a1) {
  __shared__ int s_blk[8][16], s_m[8][16];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * 8 + warp;
  pdl_wait();
  pdl_trigger();
  if (t >= T) return;
  if (lane < k) {
    const int d = tile_row[static_cast<size_t>(t) * k + lane];
    s_blk[warp][lane] = d >> 7;
    s_m[warp][lane] = d & 127;
  }
  __syncwarp();
  const int nb = H / 32, k_tiles = H / 128;
  for (int b0 = 0; b0 < nb; b0 += 32) {
    const int b = b0 + lane;
    const bool active = b < nb;  // whole quads are active or not
    uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sc = 0;
    if (active) {
      float v[32];
      load_block32_bf16(x, t, H, b, v);
      sc = quant_block32_mx(v, c);
    }
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
    const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
    if (!active) continue;
    for (int j = 0; j < k; ++j) {
      const int blk = s_blk[warp][j], m = s_m[warp][j];
      st_act_pair(a1, blk, k_tiles, b >> 2, m, (b & 3) * 2, c);
      if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(a1 + sf_atom_offset(blk, k_tiles, m, b)) = word;
    }
  }
}

cudaError_t launch_quant_a1_mx(const uint16_t* x, const int32_t* tile_row, int T, int H, int k, uint8_t* a1,
                               cudaStream_t s) {
  if (T >= 256)
    return launch_pdl(quant_a1_mx_wide_kernel, dim3((T + 7) / 8), dim3(256), 0, s, x, tile_row, T, H, k, a1);
  const int64_t threads = static_cast<int64_t>(T) * (H / 32);
  return launch_pdl(quant_a1_mx_kernel, dim3(static_cast<unsigned>((threads + 127) / 128)), dim3(128), 0, s, x,
                    tile_row, T, H, k, a1);
}

cudaError_t launch_chunk_hist(const int32_t* ids, int T, int k, int E, int32_t* chunk_counts, cudaStream_t s) {
  const int n_chunks = (T + kChunkTokens - 1) / kChunkTokens;
  return launch_pdl(chunk_hist_kernel, dim3(n_chunks), dim3(256), E * sizeof(int32_t), s, ids, T, k, E,
                    chunk_counts);
}

cudaError_t launch_scan(const int32_t* chunk_counts, int n_chunks, int E, int32_t* chunk_base, int32_t* offsets,
                        int32_t* sf_block, MBlock* mblocks, int32_t* num_mblocks, uint32_t* sched, int sched_n,
                        BlockScales bs, cudaStream_t s) {
  const int threads = ((E + 31) / 32) * 32;
  return launch_pdl(scan_kernel, dim3(1), dim3(threads), 0, s, chunk_counts, n_chunks, E, chunk_base, offsets,
                    sf_block, mblocks, num_mblocks, sched, sched_n, bs);
}

cudaError_t launch_scatter(const int32_t* ids, const int32_t* chunk_base, const int32_t* offsets,
                           const int32_t* sf_block, int T, int k, int E, int32_t* perm_src, int32_t* inv,
                           int32_t* tile_row, cudaStream_t s) {
  const int n_chunks = (T + kChunkTokens - 1) / kChunkTokens;
  const size_t smem = static_cast<size_t>(16) * E * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(scatter_kernel, dim3(n_chunks), dim3(256), smem, s, ids, chunk_base, offsets, sf_block, T, k, E,
                    perm_src, inv, tile_row);
}

cudaError_t launch_quant_a1(const uint16_t* x, const int32_t* tile_row, int T, int H, int k, float alpha, uint8_t* a1,
                            cudaStream_t s) {
  if (T >= 256)
    return launch_pdl(quant_a1_wide_kernel, dim3((T + 7) / 8), dim3(256), 0, s, x, tile_row, T, H, k, alpha, a1);
  const int64_t threads = static_cast<int64_t>(T) * (H / 16);
  return launch_pdl(quant_a1_kernel, dim3(static_cast<unsigned>((threads + 127) / 128)), dim3(128), 0, s, x, tile_row,
                    T, H, k, alpha, a1);
}

}  // namespace beam
