// Routing of a small batch (T <= 16 tokens, E <= 256 experts) in one launch: router
// logits, top-k + renormalise, histogram, scan, permutation and the 128-row work blocks.
//
// Phase 1 (every CTA): CTA (g, s) owns experts [8g, 8g + 8) (one warp each) and slice s of
// the S slices of H.  Its W_r row slices (constant: loaded before the wait for the previous
// kernel) and the x slice (T x H/S BF16) arrive in shared memory by bulk copies, one per
// row; each warp dots every token with its row slice in FP32 and a warp reduction gives one
// partial logit per (token, expert), stored to part[S][T][E].  Splitting H keeps each
// CTA's share of W_r and of x small, so 128 CTAs (E = 256, S = 4) stream W_r at once.
// Phase 2 (the last CTA to finish, found with an atomic counter after a release fence):
// one bulk copy brings every partial; logit = sum of the S partials in slice order, top-k
// per token (one warp per token), then
// the histogram, the prefix sums and the stable permutation for the whole batch, as
// routing.cu does in three launches for large batches.  The counter is reset by that CTA,
// ready for the next launch, and so are the tile scheduler words of the expert GEMM.
// Router (5120 -> 256 experts, FP32): vLLM PR "Day-0 support for Reflection's Beam-1.0",
// section "Status"; news article "vLLM adds day-zero Reflection Beam serving", section
// "Agents worked on the serving path".  8 of 256 experts: recipe
// "reflection/Beam-1.0-501B-A23B", section "Overview".
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace beam {

constexpr int kSmallExpertsPerCta = 8;                   // one warp per expert
// plus one warp whose lane 0 issues every bulk copy: a thread that issues copies runs its
// warp's math several times slower afterwards, so the copy issuer computes nothing
constexpr int kSmallThreads = (kSmallExpertsPerCta + 1) * 32;
constexpr int kCopyThread = kSmallExpertsPerCta * 32;
constexpr int kSmallMaxF4 = 16;                          // 16-byte W pieces per lane: H / S <= 2048

// Number of H slices: the largest S in {4, 2, 1} whose slice is a whole number of
// 512-byte warp rows (32 lanes x 4 floats) and at most kSmallMaxF4 of them; 0 = unsupported.
int route_small_slices(int H) {
  for (int S = 4; S >= 1; S >>= 1)
    if (H % (S * 128) == 0 && H / S / 128 <= kSmallMaxF4) return S;
  return 0;
}

// Dynamic shared memory: phase 1 holds the CTA's W_r row slices and the x slice, phase 2
// (last CTA) all partial logits.
static size_t route_small_smem(int T, int H, int E) {
  const int S = route_small_slices(H), Hs = H / S;
  const size_t p1 = static_cast<size_t>(kSmallExpertsPerCta) * Hs * 4 + static_cast<size_t>(T) * Hs * 2;
  const size_t p2 = static_cast<size_t>(S) * T * E * 4;
  return p1 > p2 ? p1 : p2;
}

template <int MAXT>
__global__ void __launch_bounds__(kSmallThreads) route_small_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ w, int T, int H, int E, int k, int S,
    float* __restrict__ part, int32_t* __restrict__ ids, float* __restrict__ wout, int32_t* __restrict__ offsets,
    int32_t* __restrict__ sf_block, MBlock* __restrict__ mblocks, int32_t* __restrict__ num_mblocks,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, int32_t* __restrict__ tile_row,
    unsigned int* __restrict__ done_counter, uint32_t* __restrict__ sched, int sched_n, BlockScales bs,
    uint32_t* __restrict__ err) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[3];  // W slices, x slice, partial logits
  __shared__ int s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hs = blockIdx.x % S, g = blockIdx.x / S;
  const int Hs = H / S, h0 = hs * Hs;
  const int nf4 = Hs / 128;
  const int e0 = g * kSmallExpertsPerCta, n_e = min(kSmallExpertsPerCta, E - e0);
  float* ws = reinterpret_cast<float*>(smem);                                              // [8][Hs] FP32
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + kSmallExpertsPerCta * Hs * 4);         // [T][Hs] BF16
  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // ---------------------------------------------------------------- phase 1: partial logits
  // Each slice row is one bulk copy.  The router weights are constant: they stream before
  // the wait for the previous kernel in the stream; x after it.
  if (tid == kCopyThread) {
    mbar_arrive_expect_tx(&bars[0], static_cast<uint32_t>(n_e * Hs * 4));
    for (int q = 0; q < n_e; ++q)
      bulk_load(ws + q * Hs, w + static_cast<size_t>(e0 + q) * H + h0, Hs * 4, &bars[0]);
  }
  pdl_wait();
  pdl_trigger();
  if (tid == kCopyThread) {
    mbar_arrive_expect_tx(&bars[1], static_cast<uint32_t>(T * Hs * 2));
    for (int t = 0; t < T; ++t) bulk_load(xs + t * Hs, x + static_cast<size_t>(t) * H + h0, Hs * 2, &bars[1]);
  }
  if (warp < n_e) {
    // every lane leaves the polling loop on its own: reconverge before the warp-wide math
    const bool ok_w = mbar_wait_bounded(&bars[0], 0, &s_abort);
    const bool ok = mbar_wait_bounded(&bars[1], 0, &s_abort) && ok_w;
    __syncwarp();
    if (!ok) {
      if (lane == 0) atomicOr(err, kErrTimeoutProducer);
    } else {
    // All tokens at once: one W piece per step, then MAXT independent FMA chains (rows
    // past T repeat row 0 and are dropped), so the smem loads and FMAs overlap.
    const float4* wr = reinterpret_cast<const float4*>(ws + warp * Hs);
    float acc[MAXT];
#pragma unroll
    for (int t = 0; t < MAXT; ++t) acc[t] = 0.0f;
#pragma unroll 2
    for (int i = 0; i < nf4; ++i) {
      const float4 wq = wr[lane + 32 * i];
#pragma unroll
      for (int t = 0; t < MAXT; ++t) {
        const int tt = t < T ? t : 0;
        const uint2 xv = reinterpret_cast<const uint2*>(xs + tt * Hs)[lane + 32 * i];
        acc[t] = fmaf(bf16_bits_to_f32(xv.x & 0xFFFFu), wq.x, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.x >> 16), wq.y, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.y & 0xFFFFu), wq.z, acc[t]);
        acc[t] = fmaf(bf16_bits_to_f32(xv.y >> 16), wq.w, acc[t]);
      }
    }
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
    }
    if (lane < T) {  // lane t stores token t's partial (selected without dynamic indexing)
      float mine = acc[0];
#pragma unroll
      for (int t = 1; t < MAXT; ++t)
        if (lane == t) mine = acc[t];
      part[(static_cast<size_t>(hs) * T + lane) * E + e0 + warp] = mine;
    }
    }
  }
  // ---------------------------------------------------------------- elect the last CTA
  // The barrier orders every thread's partial stores before thread 0's arrival, a release
  // at GPU scope (cumulative over them); the last arrival also acquires every earlier one's.
  __shared__ int s_last;
  __syncthreads();
  if (tid == 0) s_last = atom_add_acq_rel_gpu(done_counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;

  // ---------------------------------------------------------------- phase 2: top-k
  // All partial logits in one bulk copy (the other CTAs' stores were released before
  // their counter increment; the proxy fence orders them before this copy).
  float* ps = reinterpret_cast<float*>(smem);  // [S][T][E]
  if (tid == kCopyThread) {
    fence_proxy_async_global();
    fence_proxy_async_smem();  // phase 1's reads of this shared memory are done (barrier above)
    const uint32_t bytes = static_cast<uint32_t>(S * T * E * 4);
    mbar_arrive_expect_tx(&bars[2], bytes);
    bulk_load(ps, part, bytes, &bars[2]);
  }
  __syncwarp();
  // thread e's tensor scales of expert e, loaded while the partial logits are in flight
  const bool held = tid >= bs.e_begin && tid < bs.e_end;  // this handle has the expert's weights
  const float a_gu = held ? __ldg(bs.w_gu_alpha + (tid - bs.e_begin)) : 0.0f;
  const float a_d = held ? __ldg(bs.w_d_alpha + (tid - bs.e_begin)) : 0.0f;
  // the expert GEMM launch that follows starts from zeroed scheduler words
  for (int i = tid; i < sched_n; i += kSmallThreads) sched[i] = 0u;
  __shared__ int s_ids[kMaxSmallRouterTokens * 16];
  __shared__ int s_cnt[256];
  __shared__ int s_off[256];
  __shared__ int s_blk[256];
  __shared__ int warp_sums[33];
  for (int i = tid; i < E; i += kSmallThreads) s_cnt[i] = 0;
  if (!mbar_wait_bounded(&bars[2], 0, &s_abort)) {
    if (tid == 0) atomicOr(err, kErrTimeoutProducer);
  }
  __syncwarp();
  const int TE = T * E;
  for (int t = warp; t < T && warp < kSmallExpertsPerCta; t += kSmallExpertsPerCta) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ee = lane + 32 * i;
      float sum = 0.0f;
      // at most 4 slices (route_small_slices): unrolled, so the lane's 32 loads are in flight
      // together; the sum still runs over the slices in order
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < S) sum += ee < E ? ps[q * TE + t * E + ee] : 0.0f;
      v[i] = ee < E ? sum : -INFINITY;
    }
    warp_topk<8>(v, E, k, lane, s_ids + t * k, wout + static_cast<size_t>(t) * k);
  }
  __syncthreads();
  const int R = T * k;
  for (int i = tid; i < R; i += kSmallThreads) {
    ids[i] = s_ids[i];
    atomicAdd(&s_cnt[s_ids[i]], 1);
  }
  __syncthreads();
  // ---------------------------------------------------------------- scan and work blocks
  // One scan of three 10-bit fields (rows, blocks, blocks of held experts): every prefix of
  // each field is at most T k <= 256 rows or E + T k / 128 <= 258 blocks, below 2^10.
  const int cnt = tid < E ? s_cnt[tid] : 0;
  const int nblk = (cnt + 127) / 128;
  int total_packed;
  const int packed = block_exclusive_scan(cnt | (nblk << 10) | ((held ? nblk : 0) << 20), warp_sums, total_packed);
  const int off = packed & 1023, blk = (packed >> 10) & 1023, wbase = packed >> 20;
  const int total_rows = total_packed & 1023, total_blk = (total_packed >> 10) & 1023, total_work = total_packed >> 20;
  if (tid < E) {
    offsets[tid] = off;
    sf_block[tid] = blk;
    s_off[tid] = off;
    s_blk[tid] = blk;
    for (int i = 0; held && i < nblk; ++i) {
      MBlock m;
      m.expert = tid - bs.e_begin;
      m.row_begin = off + 128 * i;
      m.rows = min(128, cnt - 128 * i);
      m.sf_block = blk + i;
      m.scale_gu = bs.alpha_a1 * a_gu;
      m.scale_d = bs.alpha_a2 * a_d;
      m.pad[0] = m.pad[1] = 0;
      mblocks[wbase + i] = m;
    }
  }
  if (tid == 0) {
    offsets[E] = total_rows;
    sf_block[E] = total_blk;
    *num_mblocks = total_work;
  }
  if (tid < E) s_cnt[tid] = 0;  // from here: rows of each expert placed so far
  __syncthreads();
  // ---------------------------------------------------------------- permutation
  // rank of slot i = t k + j = earlier slots (a token chooses an expert once: earlier tokens)
  // with the same expert.  One warp walks the slots 32 at a time in order: lanes holding the
  // same expert rank among themselves by lane, after the count of the chunks before.
  if (warp == 0) {
    for (int i0 = 0; i0 < R; i0 += 32) {
      const int i = i0 + lane;
      const int ee = i < R ? s_ids[i] : -1 - lane;  // past R: a key no other lane holds
      const unsigned peers = __match_any_sync(0xffffffffu, ee);
      const int before = __popc(peers & ((1u << lane) - 1u));
      const int rank = (i < R ? s_cnt[ee] : 0) + before;
      __syncwarp();
      if (i < R && before == 0) s_cnt[ee] += __popc(peers);  // the lowest lane of each expert
      __syncwarp();
      if (i < R) {
        const int r = s_off[ee] + rank;
        perm[r] = i / k;
        inv[i] = r;
        tile_row[i] = (s_blk[ee] + (rank >> 7)) * 128 + (rank & 127);
      }
    }
  }
  if (tid == 0) *done_counter = 0u;
}

bool route_small_supported(int T, int H, int E, int k) {
  // partial logits move as one bulk copy: S * T * E * 4 bytes, a multiple of 16
  return T >= 1 && T <= kMaxSmallRouterTokens && E >= 1 && E <= 256 && E % 4 == 0 && k <= 16 &&
         route_small_slices(H) > 0 && route_small_smem(T, H, E) <= 160 * 1024;
}

int64_t route_small_ws_floats(int T, int H, int E) {
  return static_cast<int64_t>(route_small_slices(H)) * T * E;
}

cudaError_t launch_route_small(const uint16_t* x, const float* w, int T, int H, int E, int k, float* part,
                               int32_t* ids, float* wout, int32_t* offsets, int32_t* sf_block, MBlock* mblocks,
                               int32_t* num_mblocks, int32_t* perm, int32_t* inv, int32_t* tile_row,
                               unsigned int* done_counter, uint32_t* sched, int sched_n, BlockScales bs, uint32_t* err,
                               int* slices, cudaStream_t s) {
  const int S = route_small_slices(H);
  *slices = S;
  const size_t smem = route_small_smem(T, H, E);
  const int groups = (E + kSmallExpertsPerCta - 1) / kSmallExpertsPerCta;
  auto kernel = T <= 8 ? route_small_kernel<8> : route_small_kernel<kMaxSmallRouterTokens>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kernel, dim3(groups * S), dim3(kSmallThreads), smem, s, x, w, T, H, E, k, S, part, ids, wout,
                    offsets, sf_block, mblocks, num_mblocks, perm, inv, tile_row, done_counter, sched, sched_n, bs,
                    err);
}

}  // namespace beam
