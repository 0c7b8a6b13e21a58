// Internal launch interface of libbeam_moe (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace beam {

// One 128-row work block of an expert for the grouped GEMMs.
struct MBlock {
  int32_t expert;     // expert index
  int32_t row_begin;  // first permuted row
  int32_t rows;       // valid rows, 1..128
  int32_t sf_block;   // scale block of these rows (see the scale-block layout in beam_moe.h)
};

constexpr int kChunkTokens = 256;  // tokens per histogram / scatter chunk
constexpr int kMaxSmallRouterTokens = 16;

// ---- router (router.cu)
cudaError_t launch_router_logits(const uint16_t* x, const float* w, int T, int H, int E, float* logits,
                                 cudaStream_t s);
// H is split into router_split_count(T, H, E) slices; logits holds [splits][T][E] partial sums.
int router_split_count(int T, int H, int E);
cudaError_t launch_topk(const float* logits, int splits, int T, int E, int k, int32_t* ids, float* w,
                        cudaStream_t s);

// ---- permutation and activation quantisation (routing.cu)
cudaError_t launch_chunk_hist(const int32_t* ids, int T, int k, int E, int32_t* chunk_counts, cudaStream_t s);
cudaError_t launch_scan(const int32_t* chunk_counts, int n_chunks, int E, int32_t* chunk_base, int32_t* offsets,
                        int32_t* sf_block, MBlock* mblocks, int32_t* num_mblocks, cudaStream_t s);
cudaError_t launch_scatter(const int32_t* ids, const int32_t* chunk_base, int T, int k, int E, int32_t* perm_src,
                           int32_t* inv, cudaStream_t s);
cudaError_t launch_quant_a1(const uint16_t* x, const int32_t* ids, const int32_t* inv, const int32_t* offsets,
                            const int32_t* sf_block, int T, int H, int k, float alpha, uint8_t* a1, uint8_t* a1_sf,
                            cudaStream_t s);

// ---- weight quantiser and repacking (quant.cu)
cudaError_t launch_quantize_rows(const float* src, int64_t rows, int64_t cols, float alpha, const float* alpha_dev,
                                 uint8_t* codes, uint8_t* sf, cudaStream_t s);
cudaError_t launch_amax(const float* src, int64_t n, float* amax_bits, cudaStream_t s);
cudaError_t launch_amax_to_alpha(float* inout, cudaStream_t s);
// Gate/up: codes [E][2I][H/2] -> rows interleaved per 128-feature block (gate block then
// up block); scales -> 128-row scale blocks [E][2I/128][H/64][512].
cudaError_t launch_repack_gate_up(const uint8_t* codes, const uint8_t* sf, int E, int I, int H, uint8_t* codes_out,
                                  uint8_t* sf_out, cudaStream_t s);
// Down: codes [E][H][I/2] -> [E][H][Ip/2] (zero padded), scales -> [E][H/128][Ip/64][512].
cudaError_t launch_repack_down(const uint8_t* codes, const uint8_t* sf, int E, int I, int Ip, int H,
                               uint8_t* codes_out, uint8_t* sf_out, cudaStream_t s);

// ---- grouped NVFP4 GEMMs (gemm_nvfp4.cu)
struct GemmArgs {
  const MBlock* mblocks;
  const int32_t* num_mblocks;
  int n_tiles;        // output tiles of 256 columns per 128-row block
  int k_tiles;        // K / 256
  int n_rows_b;       // rows of B per expert
  const uint8_t* sfa; // activation scale blocks [blk][K/64][512]
  const uint8_t* sfb; // weight scale blocks [E][n_rows_b/128][K/64][512]
  const float* alpha_b;  // [E]
  float alpha_a;
  // gate/up epilogue: SwiGLU + NVFP4 of h
  uint8_t* a2;        // [rows][Ip/2]
  uint8_t* a2_sf;     // [blk][Ip/64][512]
  int a2_row_bytes;   // Ip/2
  int a2_kgroups;     // Ip/64
  float alpha_a2;
  // down epilogue: BF16 rows
  uint16_t* y;        // [rows][H]
  int y_cols;         // H
  uint32_t* err;
};
cudaError_t launch_gemm_gate_up(const CUtensorMap& map_a, const CUtensorMap& map_b, const GemmArgs& a, int grid,
                                cudaStream_t s);
cudaError_t launch_gemm_down(const CUtensorMap& map_a, const CUtensorMap& map_b, const GemmArgs& a, int grid,
                             cudaStream_t s);
size_t gemm_smem_bytes();

// ---- finalize (finalize.cu)
cudaError_t launch_finalize(const uint16_t* y, const float* w, const int32_t* inv, const uint16_t* residual,
                            const uint16_t* gamma, int T, int H, int k, float eps, uint16_t* out, cudaStream_t s);

}  // namespace beam
