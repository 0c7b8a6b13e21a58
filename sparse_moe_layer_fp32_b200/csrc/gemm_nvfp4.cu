// Grouped NVFP4 x NVFP4 GEMMs of the routed experts on the sm_100a tensor cores.
//
// NVFP4 routed experts run W4A4 on Blackwell (recipe "reflection/Beam-1.0-501B-A23B",
// section "Variants"); the experts are SwiGLU MLPs.  Two GEMMs per expert e over the rows
// routed to it (A = permuted NVFP4 activations, B = that expert's NVFP4 weights, both
// K-major):
//   gate/up: D[r][n] = A1[r] . Wgu[e][n],  K = H; epilogue h = silu(g) * u, A2 = Q(h)
//   down:    D[r][n] = A2[r] . Wd[e][n],   K = I; epilogue y = bf16(D * scale)
//
// Design (one persistent CTA per SM, 320 threads, warp-specialised):
//   warp 0      producer: per 256-wide K step, bulk copies of the A tile (the valid rows
//               of a 128-row activation tile, <= 16 KB), the expert's weight tile with its
//               scales (32 KB + 4 KB) and the A scales (2 KB) into a 4-stage shared-memory
//               ring, all landing on one mbarrier.  Activations and weights are both stored
//               as contiguous tiles already in the swizzled shared-memory order, so every
//               load is one sequential copy.
//   warp 1      TMEM owner; lane 0 issues tcgen05.cp (scales -> TMEM) and
//               tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M=128, N=256, K=64) into a
//               128x256 FP32 accumulator in TMEM, and tcgen05.commit to free stages.
//   warps 2..9  epilogue: tcgen05.ld the accumulator (each warp its 32-lane quarter and
//               one half of the columns), release it to the MMA warp at once, then do the
//               FP32 math and the stores while the next tile accumulates.
// Work items are (128-row block of one expert) x (256-column tile); the block list is
// built on the device by the permutation step, so the host never synchronises.
// Every mbarrier wait is bounded (kWaitLimitNs): on expiry the CTA sets the device error
// word, drains its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace beam {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;  // 256 FP4 values per K step (one 128-byte swizzle row)
constexpr int A_TILE_BYTES = BM * BK_BYTES;  // 16384: one activation tile in global memory
constexpr int B_BYTES = BN * BK_BYTES;       // 32768
constexpr int SFA_BYTES = 4 * 512;           // 4 K-groups of 64 values x 128 rows
constexpr int SFB_BYTES = 2 * 4 * 512;       // 2 row blocks of 128
static_assert(B_BYTES + SFB_BYTES == kTileBytes, "weight tile = B codes + B scales");
// Two ring shapes.  Stage layout: A | B | SFB | SFA (B and SFB are one contiguous weight
// tile).  Full: A holds 128 rows, 4 stages.  Small-M (batches of <= 32 tokens, so every
// expert has <= 32 rows): A holds 32 rows, which leaves room for a 5th stage of weights in
// flight.  The MMA still reads 128 rows of A; rows past the region read the stage's B bytes
// and only feed accumulator rows that are never stored.
template <int kStages, int kABytes>
struct Ring {
  static constexpr int STAGES = kStages;
  static constexpr int A_BYTES = kABytes;
  static constexpr int STAGE_BYTES = kABytes + B_BYTES + SFB_BYTES + SFA_BYTES;
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep 1024-byte alignment for the swizzle");
};
using RingFull = Ring<4, A_TILE_BYTES>;
using RingSmallM = Ring<5, 32 * BK_BYTES>;
constexpr int NUM_THREADS = 320;
constexpr int NUM_EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;     // 256 FP32 columns
constexpr uint32_t SFA_COL = 256;   // 4 K-groups x 4 columns
constexpr uint32_t SFB_COL = 288;   // 4 K-groups x 8 columns

// Instruction descriptor: E2M1 A and B (format 1), E4M3 scales (format 0), K-major
// operands, N = 256 (n_dim = N/8 at bit 17), M = 128 (m_dim = M/16 at bit 24).
constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);

enum Epilogue { kSwiGLU = 0, kStoreBF16 = 1 };

constexpr int kMaxStages = 5;
struct __align__(8) GemmSmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <class R>
static size_t ring_smem_bytes() {
  return static_cast<size_t>(R::STAGES) * R::STAGE_BYTES + sizeof(GemmSmemTail) + 1024;
}
size_t gemm_smem_bytes() { return ring_smem_bytes<RingFull>(); }

__device__ __forceinline__ float silu_times(float g, float u) { return __fdiv_rn(g, 1.0f + expf(-g)) * u; }

__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int EPI, class R>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_nvfp4_kernel(const GemmArgs args) {
  constexpr int STAGES = R::STAGES, A_BYTES = R::A_BYTES, STAGE_BYTES = R::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(smem + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->acc_full, 1);
    mbar_init(&tail->acc_empty, NUM_EPI_WARPS);
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  pdl_wait();  // the previous kernel's outputs (block list, activations) are complete
  pdl_trigger();

  const int n_tiles = args.n_tiles, k_tiles = args.k_tiles;
  const int kgroups = k_tiles * 4;
  const int total = *args.num_mblocks * n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const MBlock mb = args.mblocks[tile / n_tiles];
        const int nt = tile % n_tiles;
        const uint8_t* sfa = args.sfa + (static_cast<size_t>(mb.sf_block) * kgroups) * 512;
        const uint8_t* btile =
            args.b_tiles + (static_cast<size_t>(mb.expert) * n_tiles + nt) * k_tiles * static_cast<size_t>(kTileBytes);
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          uint8_t* ssfa = sb + B_BYTES + SFB_BYTES;
          // rows past the block's valid rows are not copied: their stale shared-memory
          // contents only reach accumulator rows that are never stored
          uint32_t a_bytes = static_cast<uint32_t>(min(BM, (mb.rows + 7) & ~7)) * BK_BYTES;
          if (a_bytes > static_cast<uint32_t>(A_BYTES)) {  // cannot happen when the host picks the ring right
            atomicOr(args.err, kErrRange);
            a_bytes = A_BYTES;
          }
          mbar_arrive_expect_tx(&tail->full[stage], a_bytes + kTileBytes + SFA_BYTES);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          bulk_load(sa, args.a_tiles + (static_cast<size_t>(mb.sf_block) * k_tiles + kt) * A_TILE_BYTES, a_bytes,
                    &tail->full[stage]);
          bulk_load(sb, btile + static_cast<size_t>(kt) * kTileBytes, kTileBytes, &tail->full[stage]);
          bulk_load(ssfa, sfa + static_cast<size_t>(kt) * 4 * 512, SFA_BYTES, &tail->full[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Copies still in flight land before this CTA may exit (bounded).
      for (int s = 0; s < STAGES; ++s)
        if ((armed >> s) & 1u) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&tail->full[s], (armed_parity >> s) & 1u))
            if (globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait_bounded(&tail->acc_empty, acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t ssfb = sb + B_BYTES;
          const uint32_t ssfa = ssfb + SFB_BYTES;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tc_cp_32x128b_x4(tmem + SFA_COL + kb * 4, sdesc_sf(ssfa + kb * 512));
            tc_cp_32x128b_x4(tmem + SFB_COL + kb * 8, sdesc_sf(ssfb + kb * 512));
            tc_cp_32x128b_x4(tmem + SFB_COL + kb * 8 + 4, sdesc_sf(ssfb + SFA_BYTES + kb * 512));
          }
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tc_mma_nvfp4(tmem + ACC_COL, sdesc_k_sw128(sa + kb * 32), sdesc_k_sw128(sb + kb * 32), kIdescNvfp4,
                         tmem + SFA_COL + kb * 4, tmem + SFB_COL + kb * 8, (kt | kb) != 0 ? 1u : 0u);
          }
          tc_commit(&tail->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tail->acc_full);
        acc_phase ^= 1;
      }
      // Every MMA this thread issued has finished before TMEM is freed (bounded).
      tc_commit(&tail->drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&tail->drain, 0))
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;           // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;       // which half of the 256 accumulator columns
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const MBlock mb = args.mblocks[tile / n_tiles];
      const int nt = tile % n_tiles;
      if (!mbar_wait_bounded(&tail->acc_full, acc_phase, abort_flag)) break;
      tc_fence_after();
      uint32_t v[4][32];
      if constexpr (EPI == kSwiGLU) {
        tmem_ld_32x32b_x32(t_lane + ACC_COL + half * 64, v[0]);
        tmem_ld_32x32b_x32(t_lane + ACC_COL + half * 64 + 32, v[1]);
        tmem_ld_32x32b_x32(t_lane + ACC_COL + 128 + half * 64, v[2]);
        tmem_ld_32x32b_x32(t_lane + ACC_COL + 128 + half * 64 + 32, v[3]);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(t_lane + ACC_COL + half * 128 + c * 32, v[c]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty);
      acc_phase ^= 1;
      if (row_in_tile >= mb.rows) continue;
      const size_t r = static_cast<size_t>(mb.row_begin + row_in_tile);
      (void)r;
      const float scale = args.alpha_a * __ldg(args.alpha_b + mb.expert);
      if constexpr (EPI == kSwiGLU) {
        const float alpha2 = args.alpha_a2;
        const float six_alpha2 = __fmul_rn(6.0f, alpha2);
        const int f0 = nt * 128 + half * 64;  // first feature of this thread's 64
        uint32_t codes[8];
        uint32_t scodes = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          float h[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = b * 16 + i;
            const float g = __uint_as_float(v[c >> 5][c & 31]) * scale;
            const float u = __uint_as_float(v[2 + (c >> 5)][c & 31]) * scale;
            h[i] = silu_times(g, u);
          }
          const uint32_t sc = quant_block16(h, alpha2, six_alpha2, codes[2 * b], codes[2 * b + 1]);
          scodes |= sc << (8 * b);
        }
        // 64 features = 32 bytes = 16-byte chunks c0, c0 + 1 of K tile f0 / 256 of the A2 tile
        const int a2_kt = f0 >> 8, c0 = (f0 & 255) >> 5;
        *reinterpret_cast<uint4*>(args.a2 + act_tile_offset(mb.sf_block, args.a2_k_tiles, a2_kt, row_in_tile, c0)) =
            make_uint4(codes[0], codes[1], codes[2], codes[3]);
        *reinterpret_cast<uint4*>(args.a2 + act_tile_offset(mb.sf_block, args.a2_k_tiles, a2_kt, row_in_tile, c0 + 1)) =
            make_uint4(codes[4], codes[5], codes[6], codes[7]);
        // the 4 scales of this K-group (features f0..f0+63) are 4 contiguous bytes
        *reinterpret_cast<uint32_t*>(args.a2_sf + sf_atom_offset(mb.sf_block, args.a2_kgroups, row_in_tile,
                                                                 f0 / 16)) = scodes;
      } else {
        uint4* dst = reinterpret_cast<uint4*>(args.y + r * args.y_cols + nt * BN + half * 128);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int c = q * 8;
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            p[i] = bf16x2_bits(__uint_as_float(v[(c + 2 * i) >> 5][(c + 2 * i) & 31]) * scale,
                               __uint_as_float(v[(c + 2 * i + 1) >> 5][(c + 2 * i + 1) & 31]) * scale);
          dst[q] = make_uint4(p[0], p[1], p[2], p[3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && tail->abort_flag) atomicOr(args.err, kErrTimeoutMma);
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

template <int EPI, class R>
static cudaError_t launch_ring(const GemmArgs& a, int grid, cudaStream_t s) {
  const size_t smem = ring_smem_bytes<R>();
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<EPI, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_nvfp4_kernel<EPI, R>, dim3(grid), dim3(NUM_THREADS), smem, s, a);
}

template <int EPI>
static cudaError_t launch_gemm(const GemmArgs& a, int grid, cudaStream_t s) {
  // With at most 32 tokens no expert has more than 32 rows.
  if (a.max_rows_per_expert <= 32) return launch_ring<EPI, RingSmallM>(a, grid, s);
  return launch_ring<EPI, RingFull>(a, grid, s);
}

cudaError_t launch_gemm_gate_up(const GemmArgs& a, int grid, cudaStream_t s) { return launch_gemm<kSwiGLU>(a, grid, s); }
cudaError_t launch_gemm_down(const GemmArgs& a, int grid, cudaStream_t s) { return launch_gemm<kStoreBF16>(a, grid, s); }

}  // namespace beam
