// Internal launch interface of libbeam_moe (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "beam_moe.h"

namespace beam {

// One 128-row work block of an expert for the grouped GEMMs.
struct alignas(32) MBlock {
  int32_t expert;     // expert index
  int32_t row_begin;  // first permuted row
  int32_t rows;       // valid rows, 1..128
  int32_t sf_block;   // scale block of these rows (see the scale-block layout in beam_moe.h)
  float scale_gu;     // alpha_a1 * alpha_gu[expert]: dequantisation of the gate/up accumulators
  float scale_d;      // alpha_a2 * alpha_d[expert]: dequantisation of the down accumulators
  int32_t pad[2];
};
// What the block-list builders need: the experts whose weights this handle holds (all of
// them, or one expert-parallel rank's range [e_begin, e_end); blocks of other experts are
// left out of the work list, their rows keep their places in the activations), and what
// fills MBlock::scale_gu / scale_d.  MBlock::expert is the index within the range.
struct BlockScales {
  const float* w_gu_alpha;  // [e_end - e_begin]
  const float* w_d_alpha;   // [e_end - e_begin]
  float alpha_a1, alpha_a2;
  int e_begin, e_end;
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

// ---- router on the tensor cores (router_tc.cu)
// Over (128-token tiles) x (slices of H) with partial logits that launch_topk sums: the
// default for batches of kRouterTcSplitMinTokens or more.  One tile per CTA with the top-k
// in its epilogue (router_tc_supported, from kRouterTcMinTokens tokens) is used once the
// split count falls to one (router_tc_split_count).
constexpr int kRouterTcMinTokens = 4096;
constexpr int kRouterTcSplitMinTokens = BEAM_MOE_ROUTER_TC_SPLIT_MIN_TOKENS;
bool router_tc_supported(int T, int H, int E, int k);
size_t router_tc_smem_bytes(int E);
cudaError_t launch_split_router(const float* w, int E, int H, uint16_t* out, cudaStream_t s);
// map_x: x [T][H] BF16, boxes 32 x 128 with the 64-byte swizzle; w_tiles: the split router
// weights from launch_split_router.  Writes logits [T][E], ids / w [T][k].
// Tokens per CTA (128 or 256) for a batch of T; also the row count of the x tensor map's box.
int router_tc_tokens_per_cta(int T, int num_sms);
// splits > 1: grid (token tiles) x (splits slices of H), partial logits [splits][T][E] into
// `logits`, no top-k (launch_topk sums the slices and selects).  first_token (a multiple of
// tokens_per_cta): where these T tokens start in a batch routed in parts; the FP32
// summation order of a token's logits depends only on its place in that batch.
cudaError_t launch_router_tc(const CUtensorMap& map_x, int tokens_per_cta, const uint16_t* w_tiles, int T, int H,
                             int E, int k, float* logits, int32_t* ids, float* wout, uint32_t* err, cudaStream_t s,
                             int splits = 1, int first_token = 0);
bool router_tc_split_supported(int H, int E, int k);
// The sliced form for a batch of T: tokens per CTA (128 or 256) and slices of H.
struct RouterTcPlan {
  int tokens, splits;
};
RouterTcPlan router_tc_split_plan(int T, int H, int num_sms);
int router_tc_split_count(int T, int H, int num_sms);

// ---- routing of a small batch in one launch (route_small.cu)
bool route_small_supported(int T, int H, int E, int k);
int64_t route_small_ws_floats(int T, int H, int E);  // partial logits [S][T][E]
// part: [S][T][E] partial logits over S slices of H; *slices = S.
cudaError_t launch_route_small(const uint16_t* x, const float* w, int T, int H, int E, int k, float* part,
                               int32_t* ids, float* wout, int32_t* offsets, int32_t* sf_block, MBlock* mblocks,
                               int32_t* num_mblocks, int32_t* perm, int32_t* inv, int32_t* tile_row,
                               unsigned int* done_counter, uint32_t* sched, int sched_n, BlockScales bs, uint32_t* err,
                               int* slices, cudaStream_t s);

// ---- permutation and activation quantisation (routing.cu)
cudaError_t launch_chunk_hist(const int32_t* ids, int T, int k, int E, int32_t* chunk_counts, cudaStream_t s);
// Also zeroes sched[0, sched_n), the tile scheduler words of the expert GEMM launch.
cudaError_t launch_scan(const int32_t* chunk_counts, int n_chunks, int E, int32_t* chunk_base, int32_t* offsets,
                        int32_t* sf_block, MBlock* mblocks, int32_t* num_mblocks, uint32_t* sched, int sched_n,
                        BlockScales bs, cudaStream_t s);
// tile_row[t][j] = 128 x activation block + row within it, for slot (t, j).
cudaError_t launch_scatter(const int32_t* ids, const int32_t* chunk_base, const int32_t* offsets,
                           const int32_t* sf_block, int T, int k, int E, int32_t* perm_src, int32_t* inv,
                           int32_t* tile_row, cudaStream_t s);
// A1 = Q(x) into the activation units: [blk][H/256][18432], codes then scales (common.cuh).
cudaError_t launch_quant_a1(const uint16_t* x, const int32_t* tile_row, int T, int H, int k, float alpha, uint8_t* a1,
                            cudaStream_t s);

// ---- weight quantiser and repacking (quant.cu)
// Contiguous weight tiles of the grouped GEMMs: 256 rows x 256 K values of codes in the
// swizzled shared-memory order, then their scales (see repack_tiles_kernel).
constexpr int kTileCodeBytes = 256 * 128;
constexpr int kTileSfBytes = 2 * 4 * 512;
constexpr int kTileBytes = kTileCodeBytes + kTileSfBytes;  // 36864
// rows_per_e % 256 == 0; K = logical contraction size, Kp = K rounded up to 256 (zero pad).
// interleave_inter != 0: gate/up rows, interleaved per 128 features (inter = I).
cudaError_t launch_repack_tiles(const uint8_t* codes, const uint8_t* sf, int E, int rows_per_e, int K, int Kp,
                                int interleave_inter, uint8_t* dst, cudaStream_t s);
cudaError_t launch_quantize_rows(const float* src, int64_t rows, int64_t cols, float alpha, const float* alpha_dev,
                                 uint8_t* codes, uint8_t* sf, cudaStream_t s);
cudaError_t launch_amax(const float* src, int64_t n, float* amax_bits, cudaStream_t s);
cudaError_t launch_amax_to_alpha(float* inout, cudaStream_t s);
// ---- MXFP8 experts (quant.cu, routing.cu, gemm_experts.cu)
// Weight tiles: 256 rows x 128 K values (E4M3, one byte each) in the same swizzled order
// as the NVFP4 code tiles, then 2 x 512 bytes of UE8M0 scales (4 per row: one per 32).
constexpr int kMxTileSfBytes = 2 * 512;
constexpr int kMxTileBytes = kTileCodeBytes + kMxTileSfBytes;  // 33792
// K % 128 == 0 (no padding).
cudaError_t launch_repack_tiles_mx(const uint8_t* codes, const uint8_t* sf, int E, int rows_per_e, int K,
                                   int interleave_inter, uint8_t* dst, cudaStream_t s);
cudaError_t launch_quantize_rows_mx(const float* src, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* sf,
                                    cudaStream_t s);
// A1 = MX(x) into the activation units: [blk][H/128][16896], 16384 code bytes then a
// 512-byte scale atom per K step.
cudaError_t launch_quant_a1_mx(const uint16_t* x, const int32_t* tile_row, int T, int H, int k, uint8_t* a1,
                               cudaStream_t s);

// ---- grouped NVFP4 GEMMs, gate/up and down in one launch (gemm_experts.cu)
// Activations are units of one K step, [blk][K/256][16384 code bytes, then 128 rows x 16
// scales] (act_tile_offset, sf_chunk_offset); weight tiles are [E][n_tiles][K/256][kTileBytes].
struct ExpertGemmArgs {
  const MBlock* mblocks;
  const int32_t* num_mblocks;
  int max_rows_per_expert;  // an upper bound (the number of tokens) used to pick the ring shape
  // gate/up: K = H, 256 B rows per output tile = 128 gate + 128 up features
  int gu_n_tiles;           // I / 128
  int gu_k_tiles;           // H / 256
  const uint8_t* a1;        // activation units, codes and scales
  const uint8_t* w_gu;
  // SwiGLU + NVFP4 epilogue output, the down GEMM's A operand (K = Ip)
  uint8_t* a2;               // activation units, codes and scales
  float alpha_a2;
  // down: K = Ip
  int d_n_tiles;            // H / 256
  int d_k_tiles;            // Ip / 256
  const uint8_t* w_d;
  uint16_t* y;              // [rows][H] BF16
  int y_cols;               // H
  // [0]: next tile to claim; [1 + b]: gate/up epilogue warps done on block b.
  // sched_words(nblk_max) words, zeroed by the routing kernel (two or more launches back).
  uint32_t* sched;
  uint32_t* err;
  // Expert parallelism: rows delivered into each block by the ranks (release, system scope);
  // a gate/up tile's activations are read once its block's count reaches the block's rows.
  // Null otherwise.
  const uint32_t* arrivals;
};
inline int64_t sched_words(int64_t nblk_max) { return 1 + nblk_max; }
cudaError_t launch_gemm_experts(const ExpertGemmArgs& a, int grid, cudaStream_t s);
// The same GEMMs with MXFP8 operands: K tiles of 128 values (gu_k_tiles = H / 128,
// d_k_tiles = I / 128), weight tiles of kMxTileBytes, scales [blk][K/128][512], and the
// SwiGLU epilogue writes A2 = MX(h).  alpha_a2 is unused.
cudaError_t launch_gemm_experts_mx(const ExpertGemmArgs& a, int grid, cudaStream_t s);

// ---- tensor parallel finalize fused with its all-reduce (finalize_tp.cu)
// Exchange region of a tensor-parallel rank: kTpHeaderBytes of flags (u32 slot q = the last
// epoch rank q published its partial m; slot kTpRowSlot + q = the last epoch rank q
// published its finished rows), two buffers of [max_tokens][H] FP32 partial m (epoch
// parity), then [max_tokens][H] BF16 finished rows (the two-shot form).  Expert-parallel
// regions share the header and TpGroup; their body is EpLayout below.
constexpr int kMaxTpRanks = 16;
constexpr size_t kTpHeaderBytes = 1024;
constexpr int kTpRowSlot = 4 * kMaxTpRanks;
// The two-shot all-reduce from BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS tokens on by default (every
// rank's slice is then non-empty for any world <= kMaxTpRanks, since T >= world^2).
struct TpGroup {
  uint8_t* const* regions;  // device array: every rank's region as mapped in this process
  uint8_t* own;             // this rank's region (regions[rank])
  int rank, world;
  size_t buf_floats;        // floats per partial buffer: max_tokens * H
};
// Partial m over the slots whose expert lies in [e_begin, e_end) (all of them under TP).
cudaError_t launch_tp_partial(const uint16_t* y, const float* w, const int32_t* inv, const int32_t* ids, int e_begin,
                              int e_end, int T, int H, int k, const TpGroup& g, uint32_t epoch, unsigned int* counter,
                              cudaStream_t s);
// Tokens of a rank's slice in the two-shot form: ceil(T / world).
int tp_slice_tokens(int T, int world);
// One-shot: out[t] for every t < T.  Two-shot: out[t] for this rank's slice only, also stored
// into its row buffer and published (counter: the CTA arrivals of this step).
cudaError_t launch_tp_reduce(const uint16_t* residual, const uint16_t* gamma, int T, bool two_shot, int H, float eps,
                             const TpGroup& g, uint32_t epoch, uint16_t* out, uint32_t* err, unsigned int* counter,
                             cudaStream_t s);
// Two-shot: the other ranks' finished rows into out, after a bounded wait for their flags.
cudaError_t launch_tp_gather(int T, int H, const TpGroup& g, uint32_t epoch, uint16_t* out, uint32_t* err, int grid,
                             cudaStream_t s);

// ---- expert parallelism: dispatch of routed rows, combine of expert outputs (expert_parallel.cu)
// Flag slots of the region header: rank q's counts of the epoch published / its expert
// outputs for the epoch returned.
constexpr int kEpCountSlot = 2 * kMaxTpRanks;
constexpr int kEpReturnSlot = 3 * kMaxTpRanks;
// Byte offsets in an expert-parallel rank's region (after the 1 KB flag header).
struct EpLayout {
  size_t counts;    // int32 [kMaxTpRanks][E]: rows source rank s routes to expert e
  size_t arrivals;  // u32 [nblk]: rows delivered into each 128-row block of this rank's experts
  size_t origin;    // int32 [rows]: source rank << 24 | source slot t k + j of each received row
  size_t a1;        // activation units (codes and scales) of the received rows, the GEMM layout
  size_t ret;       // BF16 [max_tokens][k][H]: this rank's slots' expert outputs, returned
  size_t bytes;     // the whole region
  int nblk;         // blocks the arrival counters cover
  int rows;         // rows of origin and of the returned rows (max_tokens k)
};
// Where source-rank rows of expert e go: destination rank, its permuted row of this rank's
// first row of e, the block of the destination's first row of e, and the rows of e that
// lower ranks send (this rank's rows of e start after them).
struct EpDest {
  int32_t rank, row0, blk0, pre;
};
// Zeroes this rank's arrival counters, then publishes its expert counts (offsets[e + 1] -
// offsets[e]) into every rank's count matrix and sets its count flag (release, system scope).
cudaError_t launch_ep_counts(const int32_t* offsets, int E, const TpGroup& g, const EpLayout& lay, uint32_t epoch,
                             cudaStream_t s);
// Waits (bounded) for every rank's counts, then: this rank's block list over its experts
// (mblocks, num_mblocks, scheduler words zeroed), its received row count, and dst[e] for
// every expert (where this rank's rows of e go).
cudaError_t launch_ep_layout(const TpGroup& g, const EpLayout& lay, int E, BlockScales bs, MBlock* mblocks,
                             int32_t* num_mblocks, uint32_t* sched, int sched_n, EpDest* dst, int32_t* own_rows,
                             uint32_t epoch, uint32_t* err, cudaStream_t s);
// Quantises this rank's tokens once (A1 = Q(x), NVFP4 or MXFP8) and stores each slot's row
// into the activation tiles of its expert's rank (peer stores), its origin, then adds the
// row to that block's arrival counter (release, system scope).
cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* inv, const int32_t* offsets,
                               const EpDest* dst, int T, int H, int k, int fmt, float alpha, const TpGroup& g,
                               const EpLayout& lay, cudaStream_t s);
// Returns every received row's expert output to its source slot (peer stores), then sets
// this rank's return flag in every rank's region (release, system scope).
cudaError_t launch_ep_combine(const uint16_t* y, const int32_t* own_rows, int H, const TpGroup& g,
                              const EpLayout& lay, uint32_t epoch, unsigned int* counter, int grid, cudaStream_t s);
// Waits (bounded) until every rank returned this epoch's rows; lets its dependents start
// only when it ends.
cudaError_t launch_ep_wait_returned(const TpGroup& g, uint32_t epoch, uint32_t* err, cudaStream_t s);

// ---- finalize (finalize.cu)
// next_x != nullptr also writes the next sublayer's pre-norm of out: bf16(out * rinv * next_gamma).
// form_T (> 0) picks the kernel form as for a batch of that many tokens (the forms sum a
// row's squares in different orders), so a batch run in parts gives the whole batch's bits.
cudaError_t launch_finalize(const uint16_t* y, const float* w, const int32_t* inv, const uint16_t* residual,
                            const uint16_t* gamma, int T, int H, int k, float eps, uint16_t* out, uint16_t* next_x,
                            const uint16_t* next_gamma, float next_eps, uint32_t* err, cudaStream_t s,
                            int form_T = 0);

}  // namespace beam
