// Router of batches above 16 tokens on the sm_100a tensor cores, at FP32-class accuracy.
//
// The router is a GEMM from hidden 5120 to 256 expert logits computed in FP32 (vLLM PR
// "Day-0 support for Reflection's Beam-1.0", section "Status"; news article "vLLM adds
// day-zero Reflection Beam serving", section "Agents worked on the serving path").  At
// prefill sizes (2 T H E = 43 GFLOP at T = 16384) FP32 FFMA would cost more than the NVFP4
// expert GEMMs, so the FP32 weights are split once, exactly, into three BF16 parts
//   W = W_hi + W_mid + W_lo   (W_hi = bf16(W), W_mid = bf16(W - W_hi), W_lo = bf16(rest);
//                              the remainder left over is below 2^-27 |W|)
// and x (BF16) times each part is an exact product, accumulated in FP32 by
// tcgen05.mma.kind::f16 in TMEM.  The result differs from an FP32 FFMA GEMM only in the
// order of the FP32 additions.
//
// One CTA per 128 x HALVES tokens (HALVES = 1 or 2): warp 0 fills a 4-stage (3-stage) ring,
// per 32-wide K step with the x tile (128 HALVES x 32 BF16, TMA, 64-byte swizzle) and the
// three weight tiles (3 x E x 32 BF16, one bulk copy: the split weights are stored
// pre-tiled in that swizzled order); warp 1 owns TMEM (one accumulator of E columns per
// 128 tokens) and issues 2 x 3 x HALVES MMAs (M = 128, N = E, K = 16) per stage.  Every CTA
// streams the whole 7.9 MB weight split; two halves per CTA halve that traffic per token,
// which pays once a batch needs more than one wave of 128-token CTAs (measured: 0.31 vs
// 0.41 ms at 32K tokens, 0.41 vs 0.36 ms at 16K).  Warps 2..(4 HALVES + 1) read their
// token's E logits from TMEM, keep a running top-k (larger logit first, equal logits ->
// lower expert index), write the logits, the chosen ids and the renormalised weights
// (softmax over the chosen logits = p_j / sum_chosen p).
//
// The default form (every batch up to ~37,900 tokens on 148 SMs): the grid is (128-token
// tiles) x (S slices of H), each CTA runs its slice's K steps only and writes its FP32
// partial logits to [S][T][E]; the top-k kernel of the SIMT router then sums the S slices in
// order and selects.  Each CTA then streams a short contiguous stretch of the weight split
// instead of all of it, and the grid fills the SMs (one wave of CTAs below 4096 tokens, two
// above): measured 81 vs 323 us at 4096 tokens and 160 vs 347 us at 16K against one tile per
// CTA.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace beam {

constexpr int RT_MMA_M = 128;
constexpr int RT_BK = 32;  // BF16 values per K step = one 64-byte swizzle row
constexpr int RT_MAX_STAGES = 4;
template <int HALVES>
struct RtShape {
  static constexpr int BM = HALVES * RT_MMA_M;  // tokens per CTA
  static constexpr int STAGES = HALVES == 1 ? 4 : 3;
  static constexpr int A_BYTES = BM * 64;
  static constexpr int THREADS = (2 + 4 * HALVES) * 32;
};

struct __align__(8) RouterSmemTail {
  uint64_t full[RT_MAX_STAGES];
  uint64_t empty[RT_MAX_STAGES];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

template <int HALVES>
static size_t router_tc_smem(int E) {
  using S = RtShape<HALVES>;
  return S::STAGES * (S::A_BYTES + 3 * static_cast<size_t>(E) * 64) + sizeof(RouterSmemTail) + 1024;
}
size_t router_tc_smem_bytes(int E) { return std::max(router_tc_smem<1>(E), router_tc_smem<2>(E)); }

// E columns of TMEM rounded up to a power of two >= 32
static __host__ __device__ uint32_t tmem_cols_for(int E) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(E)) c <<= 1;
  return c;
}

template <int HALVES>
__global__ void __launch_bounds__(RtShape<HALVES>::THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap map_x, const uint8_t* __restrict__ w_tiles, int T,
                     int H, int E, int k, float* __restrict__ logits, int32_t* __restrict__ ids,
                     float* __restrict__ wout, uint32_t* __restrict__ err, int splits, int tile_base) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int RT_BM = RtShape<HALVES>::BM, RT_STAGES = RtShape<HALVES>::STAGES, RT_A_BYTES = RtShape<HALVES>::A_BYTES;
  const int stage_bytes = RT_A_BYTES + 3 * E * 64;
  RouterSmemTail* tail = reinterpret_cast<RouterSmemTail*>(smem + RT_STAGES * stage_bytes);
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tcols = tmem_cols_for(E);  // per accumulator; two are allocated
  if (threadIdx.x == 0) {
    for (int s = 0; s < RT_STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->acc_full, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, HALVES * tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  pdl_wait();
  pdl_trigger();
  const int m0 = blockIdx.x * RT_BM;
  // this CTA's K steps: [k_lo, k_lo + k_tiles) of H / RT_BK (all of them when splits == 1)
  const int k_all = H / RT_BK;
  const int k_per = (k_all + splits - 1) / splits;
  const int k_lo = static_cast<int>(blockIdx.y) * k_per;
  const int k_tiles = max(0, min(k_per, k_all - k_lo));
  // Every CTA reads the same weight tiles; starting each CTA at a different K step keeps
  // them from all hitting the same L2 lines at once.  Only the FP32 summation order changes
  // with the start, which follows the tile's index in the whole batch (tile_base: this
  // launch's first tile), so a batch routed in parts sums every token's logits alike.
  const int k_start = k_tiles > 0 ? (tile_base + static_cast<int>(blockIdx.x)) % k_tiles : 0;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&map_x);
      int stage = 0;
      uint32_t phase = 0, armed = 0, armed_parity = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1, abort_flag)) break;
        uint8_t* sa = smem + stage * stage_bytes;
        mbar_arrive_expect_tx(&tail->full[stage], static_cast<uint32_t>(stage_bytes));
        armed |= 1u << stage;
        armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
        const int kk = k_lo + (kt + k_start) % k_tiles;
        tma_load_2d(sa, &map_x, &tail->full[stage], kk * RT_BK, m0);
        bulk_load(sa + RT_A_BYTES, w_tiles + static_cast<size_t>(kk) * 3 * E * 64, 3 * E * 64, &tail->full[stage]);
        if (++stage == RT_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      for (int s = 0; s < RT_STAGES; ++s)
        if ((armed >> s) & 1u) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&tail->full[s], (armed_parity >> s) & 1u))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // BF16 x BF16 -> FP32, K-major A and B, N = E, M = 128
      const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(E) >> 3) << 17) |
                             ((RT_MMA_M >> 4) << 24);
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * stage_bytes);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
#pragma unroll
          for (int p = 0; p < 3; ++p) {
            const uint64_t bdesc = sdesc_k_sw64(sa + RT_A_BYTES + p * E * 64 + kb * 32);
#pragma unroll
            for (int h = 0; h < HALVES; ++h)  // tokens 128 h .. 128 h + 127: rows start 128 x 64 bytes in
              tc_mma_bf16(tmem + h * tcols, sdesc_k_sw64(sa + h * RT_MMA_M * 64 + kb * 32), bdesc, idesc,
                          (kt | kb | p) != 0);
          }
        tc_commit(&tail->empty[stage]);
        if (++stage == RT_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      // an empty slice (k_tiles == 0: the splits do not divide H evenly) issued nothing; its
      // epilogue writes zeros
      tc_commit(&tail->acc_full);  // also fires after an abort, once the issued MMAs finish
      // every issued MMA has finished before TMEM can be freed (bounded)
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&tail->acc_full, 0))
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // which accumulator (128-token half)
    const int t = m0 + half * RT_MMA_M + quarter * 32 + lane;
    const bool ok = mbar_wait_bounded(&tail->acc_full, 0, abort_flag);
    tc_fence_after();
    float best_v[16];
    int best_e[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      best_v[j] = -INFINITY;
      best_e[j] = 0x7fffffff;
    }
    float thr = -INFINITY;  // current k-th largest
    const uint32_t t_lane = tmem + half * tcols + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool partial = splits > 1;  // write this slice's partial logits only
    for (int c0 = 0; c0 < E; c0 += 32) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(t_lane + c0, v);  // E % 16 == 0: columns past E are never used
      tmem_ld_wait();
      if (!ok || t >= T) continue;
      if (k_tiles == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0u;  // the accumulator was never written
      }
      const int ncols = min(32, E - c0);
      float* lrow = logits + (static_cast<size_t>(blockIdx.y) * T + t) * E + c0;
      if (ncols == 32) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(lrow)[i] =
              make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                          __uint_as_float(v[4 * i + 3]));
      } else {
        for (int i = 0; i < ncols; ++i) lrow[i] = __uint_as_float(v[i]);
      }
      if (partial) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float cv = __uint_as_float(v[i]);
        if (i >= ncols || !(cv > thr)) continue;  // equal to the k-th: the lower index already there wins
        int ce = c0 + i;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < k && cv > best_v[j]) {
            const float tv = best_v[j];
            const int te = best_e[j];
            best_v[j] = cv;
            best_e[j] = ce;
            cv = tv;
            ce = te;
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j == k - 1) thr = best_v[j];
      }
    }
    if (ok && t < T && !partial) {
      float z[16], sum = 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        z[j] = j < k ? expf(best_v[j] - best_v[0]) : 0.0f;
        sum += z[j];
      }
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < k) {
          ids[static_cast<size_t>(t) * k + j] = best_e[j];
          wout[static_cast<size_t>(t) * k + j] = z[j] / sum;
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && tail->abort_flag) atomicOr(err, kErrTimeoutMma);
  if (warp == 1) tmem_dealloc(tmem, HALVES * tcols);
}

// W_r [E][H] FP32 -> BF16 parts hi, mid, lo (each rounded to nearest even), stored as
// tiles [H/32][3][E rows x 64 bytes]: each 64-byte row holds 32 values of one expert, its
// four 16-byte chunks placed at chunk ^ ((row >> 1) & 3) (the 64-byte swizzle), so one
// K step of all three parts is one contiguous copy in shared-memory order.
__global__ void split_router_kernel(const float* __restrict__ w, int E, int H, uint16_t* __restrict__ out) {
  const int64_t n = static_cast<int64_t>(E) * H;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int e = static_cast<int>(i / H), h = static_cast<int>(i % H);
    const float a = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(a);
    const float r1 = a - __bfloat162float(hi);  // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);  // exact
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    const int kt = h / RT_BK, col = h % RT_BK;  // value col of the 64-byte row
    const int chunk = (col >> 3) ^ ((e >> 1) & 3), within = col & 7;
    const int64_t base = (static_cast<int64_t>(kt) * 3 * E + e) * RT_BK + chunk * 8 + within;  // in BF16 units
    const __nv_bfloat16 parts[3] = {hi, mid, lo};
#pragma unroll
    for (int p = 0; p < 3; ++p)
      out[base + static_cast<int64_t>(p) * E * RT_BK] = *reinterpret_cast<const uint16_t*>(&parts[p]);
  }
}

cudaError_t launch_split_router(const float* w, int E, int H, uint16_t* out, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(E) * H;
  split_router_kernel<<<static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 148 * 8)), 256, 0, s>>>(w, E, H,
                                                                                                       out);
  return cudaGetLastError();
}

bool router_tc_supported(int T, int H, int E, int k) {
  return T >= kRouterTcMinTokens && H % RT_BK == 0 && E % 16 == 0 && E >= 16 && E <= 256 && k <= 16 &&
         router_tc_smem_bytes(E) <= 227 * 1024;
}

bool router_tc_split_supported(int H, int E, int k) {
  return H % RT_BK == 0 && E % 16 == 0 && E >= 16 && E <= 256 && k <= 16 && router_tc_smem_bytes(E) <= 227 * 1024;
}

RouterTcPlan router_tc_split_plan(int T, int H, int num_sms) {
  // (token tiles) x (slices of H), each slice at least 4 K steps: about one wave of CTAs
  // below kRouterTcMinTokens tokens, about two from there on
  const int tiles = (T + RT_MMA_M - 1) / RT_MMA_M;
  const int max_splits = std::max(1, H / RT_BK / 4);
  const int want = T < kRouterTcMinTokens ? num_sms / tiles : (2 * num_sms + tiles - 1) / tiles;
  return RouterTcPlan{RT_MMA_M, std::max(1, std::min(want, max_splits))};
}

int router_tc_split_count(int T, int H, int num_sms) { return router_tc_split_plan(T, H, num_sms).splits; }

int router_tc_tokens_per_cta(int T, int num_sms) {
  // two halves per CTA once 128-token CTAs would need more than one wave
  return T > num_sms * RT_MMA_M ? 2 * RT_MMA_M : RT_MMA_M;
}

template <int HALVES>
static cudaError_t launch_router_tc_t(const CUtensorMap& map_x, const uint16_t* w_tiles, int T, int H, int E, int k,
                                      float* logits, int32_t* ids, float* wout, uint32_t* err, int splits,
                                      int tile_base, cudaStream_t s) {
  using S = RtShape<HALVES>;
  const size_t smem = router_tc_smem<HALVES>(E);
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<HALVES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(router_tc_kernel<HALVES>, dim3((T + S::BM - 1) / S::BM, splits), dim3(S::THREADS), smem, s,
                    map_x, reinterpret_cast<const uint8_t*>(w_tiles), T, H, E, k, logits, ids, wout, err, splits,
                    tile_base);
}

cudaError_t launch_router_tc(const CUtensorMap& map_x, int tokens_per_cta, const uint16_t* w_tiles, int T, int H,
                             int E, int k, float* logits, int32_t* ids, float* wout, uint32_t* err, cudaStream_t s,
                             int splits, int first_token) {
  if (splits < 1 || first_token % tokens_per_cta != 0) return cudaErrorInvalidValue;
  const int tile_base = first_token / tokens_per_cta;
  if (tokens_per_cta == 2 * RT_MMA_M)
    return launch_router_tc_t<2>(map_x, w_tiles, T, H, E, k, logits, ids, wout, err, splits, tile_base, s);
  if (tokens_per_cta == RT_MMA_M)
    return launch_router_tc_t<1>(map_x, w_tiles, T, H, E, k, logits, ids, wout, err, splits, tile_base, s);
  return cudaErrorInvalidValue;
}

}  // namespace beam
