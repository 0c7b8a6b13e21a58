// Expert parallelism with attention data parallelism: only the routed rows travel.
//
// The vLLM PR "Day-0 support for Reflection's Beam-1.0" (section "Status") serves Beam with
// attention data parallelism and the MegaMoE expert kernels, whose role is the expert
// all-to-all overlapped with the expert GEMMs; the recipe "reflection/Beam-1.0-501B-A23B"
// ("Overview": 8 of 256 experts; "Launching the server": expert parallel with data-parallel
// attention).  Each of W ranks holds E / W experts and its own batch.  Per forward:
//
//   phase 0  route the rank's own tokens (the single-GPU routing kernels), then
//            ep_counts: zero this rank's arrival counters, write its per-expert row counts
//            into every rank's count matrix, set its count flag (release, system scope);
//   phase 1  ep_layout: wait for every rank's counts; from the count matrix every rank
//            derives the same layout: each rank's received rows, expert-major over its
//            experts, within an expert by source rank then token, in 128-row blocks;
//            this rank's block list as a destination, and where its own rows go;
//            ep_dispatch: quantise each own token once (A1) and store each slot's row into
//            the activation tiles of its expert's rank (peer stores), with its origin,
//            then add the row to that block's arrival counter (release, system scope);
//   phase 2  the expert GEMMs over the received rows (a gate/up tile reads its block's
//            activations once the block's arrival count is complete, so the GEMMs start on
//            rows that have arrived while others are still in flight), then
//            ep_combine: every received row's expert output back to its source slot (peer
//            stores), then this rank's return flag in every rank's region;
//   phase 3  wait for every rank's return flag, then the usual finalize over the rank's own
//            tokens from the returned rows (slot order, this rank's routing weights).
//
// Buffers are reused every forward without double buffering: a rank writes into a peer's
// buffers for forward n + 1 only after it has seen that peer's counts for n + 1, which the
// peer publishes only after it has finished forward n.  On one GPU the ranks run phase by
// phase (every rank's phase p before any rank's phase p + 1); every wait is then already
// satisfied when it runs.  Every wait is bounded (kWaitLimitNs) and reports a timeout in the
// error word.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace beam {

__device__ __forceinline__ uint32_t* ep_flags(uint8_t* region) { return reinterpret_cast<uint32_t*>(region); }

// Waits until the flag holds `epoch` or later (epochs only grow; compared modulo 2^32).
__device__ __forceinline__ bool ep_wait_flag(const uint32_t* flag, uint32_t epoch) {
  const uint64_t t0 = globaltimer_ns();
  while (static_cast<int32_t>(ld_acquire_sys(flag) - epoch) < 0) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(64);
  }
  return true;
}

// ------------------------------------------------------------------ phase 0: counts
__global__ void __launch_bounds__(1024) ep_counts_kernel(const int32_t* __restrict__ offsets, int E, TpGroup g,
                                                         EpLayout lay, uint32_t epoch) {
  pdl_wait();
  pdl_trigger();
  // no rank writes this rank's counters for this epoch before it has seen the flag below
  uint32_t* arrivals = reinterpret_cast<uint32_t*>(g.own + lay.arrivals);
  for (int i = threadIdx.x; i < lay.nblk; i += blockDim.x) arrivals[i] = 0u;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t c = offsets[e + 1] - offsets[e];
    for (int q = 0; q < g.world; ++q) reinterpret_cast<int32_t*>(g.regions[q] + lay.counts)[g.rank * E + e] = c;
  }
  __syncthreads();  // every thread's stores before thread 0's (cumulative) release
  if (threadIdx.x == 0)
    for (int q = 0; q < g.world; ++q) st_release_sys(ep_flags(g.regions[q]) + kEpCountSlot + g.rank, epoch);
}

// ------------------------------------------------------------------ phase 1: layout
__global__ void __launch_bounds__(1024) ep_layout_kernel(TpGroup g, EpLayout lay, int E, BlockScales bs,
                                                         MBlock* __restrict__ mblocks, int32_t* __restrict__ num_mblocks,
                                                         uint32_t* __restrict__ sched, int sched_n,
                                                         EpDest* __restrict__ dst, int32_t* __restrict__ own_rows,
                                                         uint32_t epoch, uint32_t* __restrict__ err) {
  __shared__ int s_ok;
  __shared__ int warp_sums[33];
  __shared__ int s_rows[1025], s_blk[1025];  // exclusive scans over all experts, then the totals
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (tid == 0) s_ok = 1;
  __syncthreads();
  if (tid < g.world && !ep_wait_flag(ep_flags(g.own) + kEpCountSlot + tid, epoch)) {
    atomicOr(err, kErrTimeoutEpilogue);
    s_ok = 0;
  }
  __syncthreads();  // the waiting threads' acquires order every thread's count loads below
  const bool ok = s_ok != 0;
  const int32_t* cnt = reinterpret_cast<const int32_t*>(g.own + lay.counts);
  int total = 0, pre = 0;
  if (tid < E && ok)
    for (int sr = 0; sr < g.world; ++sr) {
      const int c = __ldcv(cnt + sr * E + tid);
      total += c;
      if (sr < g.rank) pre += c;
    }
  const int nblk = (total + 127) / 128;
  int all_rows, all_blk;
  const int xrows = block_exclusive_scan(tid < E ? total : 0, warp_sums, all_rows);
  const int xblk = block_exclusive_scan(tid < E ? nblk : 0, warp_sums, all_blk);
  if (tid < E) {
    s_rows[tid] = xrows;
    s_blk[tid] = xblk;
  }
  if (tid == 0) {
    s_rows[E] = all_rows;
    s_blk[E] = all_blk;
  }
  __syncthreads();
  const int e_loc = bs.e_end - bs.e_begin;  // every rank holds as many experts, in rank order
  if (tid < E) {
    const int d = tid / e_loc, first = d * e_loc;
    dst[tid] = EpDest{d, xrows - s_rows[first] + pre, xblk - s_blk[first], pre};
    if (tid >= bs.e_begin && tid < bs.e_end) {  // this rank's expert: its blocks
      const int base = xrows - s_rows[bs.e_begin], blk = xblk - s_blk[bs.e_begin];
      const int le = tid - bs.e_begin;
      const float sgu = bs.alpha_a1 * __ldg(bs.w_gu_alpha + le), sd = bs.alpha_a2 * __ldg(bs.w_d_alpha + le);
      for (int i = 0; i < nblk && blk + i < lay.nblk; ++i)
        mblocks[blk + i] = MBlock{le, base + 128 * i, min(128, total - 128 * i), blk + i, sgu, sd, {0, 0}};
    }
  }
  if (tid == 0) {
    const int nb = s_blk[bs.e_end] - s_blk[bs.e_begin];
    if (nb > lay.nblk) atomicOr(err, kErrRange);
    *num_mblocks = ok ? min(nb, lay.nblk) : 0;
    *own_rows = ok ? min(s_rows[bs.e_end] - s_rows[bs.e_begin], lay.rows) : 0;
  }
  for (int i = tid; i < sched_n; i += blockDim.x) sched[i] = 0u;  // the expert GEMM's scheduler words
}

// ------------------------------------------------------------------ phase 1: dispatch
// One CTA per token, one lane per 16-value (NVFP4) or 32-value (MXFP8) block of its row (a
// single step at H = 5120: every load of the row is in flight at once): the row is quantised
// once and each 16-byte chunk / scale word stored into every slot's destination; after a
// barrier, thread j publishes slot j (its origin, then a release add on its block's arrival
// counter, which covers the whole CTA's stores).
constexpr int kEpMaxK = 16;
constexpr int kEpDispatchThreads = 512;
template <bool kMx>
__global__ void __launch_bounds__(kEpDispatchThreads) ep_dispatch_kernel(
    const uint16_t* __restrict__ x, const int32_t* __restrict__ ids, const int32_t* __restrict__ inv,
    const int32_t* __restrict__ offsets, const EpDest* __restrict__ dst, int T, int H, int k, float alpha, TpGroup g,
    EpLayout lay) {
  __shared__ uint8_t* s_a1[kEpMaxK];
  __shared__ int s_blk[kEpMaxK], s_m[kEpMaxK];
  const int tid = threadIdx.x, lane = tid & 31;
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  int row = 0, blk = 0, dr = 0;
  bool in_range = false;
  if (tid < k) {
    const size_t i = static_cast<size_t>(t) * k + tid;
    const int e = ids[i];
    const EpDest o = dst[e];
    const int li = inv[i] - offsets[e];  // this token's rank among this rank's rows of e
    const int pos = o.pre + li;          // among the destination's rows of e
    row = o.row0 + li;
    blk = o.blk0 + (pos >> 7);
    dr = o.rank;
    in_range = blk < lay.nblk && dr < g.world && row < lay.rows;
    s_a1[tid] = g.regions[in_range ? dr : g.rank] + lay.a1;
    s_blk[tid] = in_range ? blk : -1;
    s_m[tid] = pos & 127;
  }
  __syncthreads();
  const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
  if constexpr (!kMx) {
    const float six_alpha = __fmul_rn(6.0f, alpha);
    const int nb = H / 16;
    // the loop bound is the same for the whole warp (blockDim is a multiple of 32): shuffles
    // below always see every lane
    for (int b0 = 0; b0 < nb; b0 += blockDim.x) {
      const int b = b0 + tid;
      const bool active = b < nb;  // whole quads are active or not (nb % 4 == 0)
      uint32_t lo = 0, hi = 0, sc = 0;
      if (active) {
        const uint4 p0 = __ldg(xr + 2 * b), p1 = __ldg(xr + 2 * b + 1);
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
        const int bj = s_blk[j], m = s_m[j];
        if (bj < 0) continue;
        *reinterpret_cast<uint4*>(s_a1[j] + act_tile_offset(bj, H / 256, b >> 4, m, (b & 15) >> 1)) =
            make_uint4(lo, hi, lo1, hi1);
        if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(s_a1[j] + sf_chunk_offset(bj, H / 256, m, b)) = word;
      }
    }
  } else {
    const int nb = H / 32, k_tiles = H / 128;
    for (int b0 = 0; b0 < nb; b0 += blockDim.x) {
      const int b = b0 + tid;
      const bool active = b < nb;
      uint32_t c[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sc = 0;
      if (active) {
        float v[32];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 p = __ldg(xr + 4 * b + q);
          const uint32_t u[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[8 * q + 2 * i] = bf16_bits_to_f32(u[i] & 0xFFFFu);
            v[8 * q + 2 * i + 1] = bf16_bits_to_f32(u[i] >> 16);
          }
        }
        sc = quant_block32_mx(v, c);
      }
      const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
      const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
      const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
      const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
      if (!active) continue;
      for (int j = 0; j < k; ++j) {
        const int bj = s_blk[j], m = s_m[j];
        if (bj < 0) continue;
        st_act_pair(s_a1[j], bj, k_tiles, b >> 2, m, (b & 3) * 2, c);
        if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(s_a1[j] + sf_atom_offset(bj, k_tiles, m, b)) = word;
      }
    }
  }
  // every thread's stores of the k rows come before each slot's origin and arrival: the
  // barrier orders them before thread j, whose release add is cumulative over them
  __syncthreads();
  if (tid < k && in_range) {
    reinterpret_cast<int32_t*>(g.regions[dr] + lay.origin)[row] = (g.rank << 24) | (t * k + tid);
    red_add_release_sys(reinterpret_cast<uint32_t*>(g.regions[dr] + lay.arrivals) + blk, 1u);
  }
}

// ------------------------------------------------------------------ phase 2: combine
// One warp per received row, grid-stride: its BF16 expert output to its source slot.
__global__ void __launch_bounds__(256) ep_combine_kernel(const uint16_t* __restrict__ y,
                                                         const int32_t* __restrict__ own_rows, int H, TpGroup g,
                                                         EpLayout lay, uint32_t epoch, uint32_t* __restrict__ counter) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  pdl_wait();
  pdl_trigger();
  const int rows = *own_rows;
  const int32_t* origin = reinterpret_cast<const int32_t*>(g.own + lay.origin);
  for (int r = blockIdx.x * 8 + warp; r < rows; r += gridDim.x * 8) {
    const int o = origin[r];
    const int src = o >> 24;
    const size_t slot = static_cast<size_t>(o & 0xFFFFFF);
    if (src < 0 || src >= g.world || slot >= static_cast<size_t>(lay.rows)) continue;  // only if a rank failed
    const uint4* sp = reinterpret_cast<const uint4*>(y + static_cast<size_t>(r) * H);
    uint4* dp = reinterpret_cast<uint4*>(g.regions[src] + lay.ret) + slot * (H / 8);
    for (int c = lane; c < H / 8; c += 32) dp[c] = sp[c];
  }
  // as tp_partial: the CTA barrier orders this CTA's stores before thread 0's release; the
  // last arrival's system-scope release of the flags carries every CTA's stores
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t done = atom_add_acq_rel_gpu(counter, 1u);
    if (done == gridDim.x - 1) {
      *counter = 0u;
      for (int q = 0; q < g.world; ++q) st_release_sys(ep_flags(g.regions[q]) + kEpReturnSlot + g.rank, epoch);
    }
  }
}

// ------------------------------------------------------------------ phase 3: wait
// One CTA; it never triggers its dependents early, so the finalize that reads the returned
// rows (some of them before its own grid-dependency wait) starts only once it has ended.
__global__ void ep_wait_returned_kernel(TpGroup g, uint32_t epoch, uint32_t* err) {
  pdl_wait();
  if (threadIdx.x < g.world && !ep_wait_flag(ep_flags(g.own) + kEpReturnSlot + threadIdx.x, epoch))
    atomicOr(err, kErrTimeoutEpilogue);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_ep_counts(const int32_t* offsets, int E, const TpGroup& g, const EpLayout& lay, uint32_t epoch,
                             cudaStream_t s) {
  return launch_pdl(ep_counts_kernel, dim3(1), dim3(1024), 0, s, offsets, E, g, lay, epoch);
}

cudaError_t launch_ep_layout(const TpGroup& g, const EpLayout& lay, int E, BlockScales bs, MBlock* mblocks,
                             int32_t* num_mblocks, uint32_t* sched, int sched_n, EpDest* dst, int32_t* own_rows,
                             uint32_t epoch, uint32_t* err, cudaStream_t s) {
  if (E > 1024) return cudaErrorInvalidValue;
  return launch_pdl(ep_layout_kernel, dim3(1), dim3(1024), 0, s, g, lay, E, bs, mblocks, num_mblocks, sched, sched_n,
                    dst, own_rows, epoch, err);
}

cudaError_t launch_ep_dispatch(const uint16_t* x, const int32_t* ids, const int32_t* inv, const int32_t* offsets,
                               const EpDest* dst, int T, int H, int k, int fmt, float alpha, const TpGroup& g,
                               const EpLayout& lay, cudaStream_t s) {
  if (k > kEpMaxK) return cudaErrorInvalidValue;
  const bool mx = fmt == BEAM_MOE_FMT_MXFP8;
  const int lanes = H / (mx ? 32 : 16);  // one lane per block of the row, whole warps, at most kEpDispatchThreads
  const int threads = std::min(kEpDispatchThreads, (lanes + 31) / 32 * 32);
  if (mx)
    return launch_pdl(ep_dispatch_kernel<true>, dim3(T), dim3(threads), 0, s, x, ids, inv, offsets, dst, T, H, k,
                      alpha, g, lay);
  return launch_pdl(ep_dispatch_kernel<false>, dim3(T), dim3(threads), 0, s, x, ids, inv, offsets, dst, T, H, k, alpha,
                    g, lay);
}

cudaError_t launch_ep_combine(const uint16_t* y, const int32_t* own_rows, int H, const TpGroup& g,
                              const EpLayout& lay, uint32_t epoch, unsigned int* counter, int grid, cudaStream_t s) {
  return launch_pdl(ep_combine_kernel, dim3(grid), dim3(256), 0, s, y, own_rows, H, g, lay, epoch, counter);
}

cudaError_t launch_ep_wait_returned(const TpGroup& g, uint32_t epoch, uint32_t* err, cudaStream_t s) {
  return launch_pdl(ep_wait_returned_kernel, dim3(1), dim3(32), 0, s, g, epoch, err);
}

}  // namespace beam
