// Grouped NVFP4 x NVFP4 GEMMs of the routed experts on the sm_100a tensor cores: the
// gate/up GEMM and the down GEMM of every expert in ONE persistent launch.
//
// NVFP4 routed experts run W4A4 on Blackwell (recipe "reflection/Beam-1.0-501B-A23B",
// section "Variants"); the experts are SwiGLU MLPs.  Two GEMMs per expert e over the rows
// routed to it (A = permuted NVFP4 activations, B = that expert's NVFP4 weights, both
// K-major):
//   gate/up: D[r][n] = A1[r] . Wgu[e][n],  K = H; epilogue h = silu(g) * u, A2 = Q(h)
//   down:    D[r][n] = A2[r] . Wd[e][n],   K = I; epilogue y = bf16(D * scale)
// The single-CTA kernel is also built for the recipe's second precision variant, FP8
// experts (same section), read as MXFP8: E4M3 operands with one UE8M0 scale per 32 values,
// tcgen05.mma.kind::mxf8f6f4, and A2 = MX(h) in the epilogue (template parameter FmtMxfp8).
//
// Work items are (128-row block of one expert) x (256-column tile).  The tile list holds
// every gate/up tile, then every down tile; CTAs claim tiles in that order from a global
// counter, so a CTA that drew cheap tiles takes more, and the down tiles of early blocks
// fill the tail of the gate/up work instead of waiting for a second launch.  A down tile
// of block b needs all of block b's A2 columns: every epilogue warp that finishes a
// gate/up tile of b publishes its stores (proxy fence, release) and bumps ready[b]; the
// producer that claimed the down tile waits (bounded) until ready[b] counts all of them,
// then reads A2 with bulk copies.  Claims are in list order and a gate/up tile never
// waits on anything, so every awaited tile is held by a running CTA: no deadlock, and no
// need for all CTAs to be resident at once.
//
// CTA layout (one persistent CTA per SM, 704 threads, warp-specialised):
//   warp 0      producer: claims tiles, publishes each tile id through a small shared
//               ring, and per 256-wide K step bulk-copies the expert's weight tile with its
//               scales (32 KB + 4 KB) and the block's activation unit (16 KB of codes, then
//               the K step's 128 rows x 16 scale bytes; MXFP8: one 512-byte atom) into the
//               stage ring, all landing on one mbarrier: two copies for a block of 128 rows,
//               and for a block of fewer rows its valid rows' codes and scales (two copies).
//               Activations and weights are both stored already in the swizzled
//               shared-memory order, so every load is one sequential copy.
//   warp 1      TMEM owner; lane 0 issues tcgen05.mma.kind::mxf4nvf4.block_scale.block16
//               (M=128, N=256, K=64) into a 128x256 FP32 accumulator in TMEM and
//               tcgen05.commit to free stages.
//   warps 2..17 epilogue: tcgen05.ld the accumulator (each warp its 32-lane quarter and
//               a quarter of the columns), release it to the MMA warp at once, then do the
//               FP32 math and the stores while the next tile accumulates.  The SwiGLU +
//               NVFP4 epilogue is the longest per-tile step at prefill, so it gets four
//               warps per SM sub-partition to hide its latencies.
//   warps 18-21 scale factors: per stage, copy the A and B scales from shared memory to that
//               stage's TMEM columns with tcgen05.st (one warp per lane quarter).  Done with
//               tcgen05.cp by the MMA thread, the 12 copies per K step took the tensor pipe
//               about as long as the 4 MMAs.
// Every wait is bounded (kWaitLimitNs): on expiry the CTA sets the device error word,
// drains its own copies and MMAs, frees TMEM and exits.
#include "common.cuh"
#include "internal.h"

namespace beam {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK_BYTES = 128;  // 256 FP4 values per K step (one 128-byte swizzle row)
constexpr int A_TILE_BYTES = BM * BK_BYTES;  // 16384: the codes of one activation unit
constexpr int B_BYTES = BN * BK_BYTES;       // 32768
constexpr int SFA_BYTES = 128 * 16;          // 128 rows x 16 scales (the K step's 256 values)
constexpr int SFB_BYTES = 2 * 4 * 512;       // 2 row blocks of 128
static_assert(B_BYTES + SFB_BYTES == kTileBytes, "weight tile = B codes + B scales");
static_assert(A_TILE_BYTES == kActCodeBytes, "activation unit codes");
//
// Operand formats.  A K step is one 128-byte swizzle row per operand row in both: 256 E2M1
// values (NVFP4: 4 MMAs of K = 64, 16 scales of 16 values per row) or 128 E4M3 values
// (MXFP8: 4 MMAs of K = 32, 4 scales of 32 values per row).  Scale bytes per K step:
struct FmtNvfp4 {
  static constexpr bool kMx = false;
  static constexpr int SFA = SFA_BYTES;    // one K-step chunk: [128 rows][16 scales]
  static constexpr int SFB = SFB_BYTES;    // 2 row halves x 4 atoms
  static constexpr int TILE = kTileBytes;  // weight tile: B codes + B scales
  static constexpr int UNIT = kActUnitNvfp4;  // activation unit: A codes + A scales
};
struct FmtMxfp8 {
  static constexpr bool kMx = true;
  static constexpr int SFA = 512;          // 1 atom: the 4 scales of a row in one 32-bit word
  static constexpr int SFB = 2 * 512;      // 2 row halves
  static constexpr int TILE = kMxTileBytes;
  static constexpr int UNIT = kActUnitMx;
};
static_assert(B_BYTES + FmtMxfp8::SFB == kMxTileBytes, "MXFP8 weight tile = B codes + B scales");
static_assert(FmtNvfp4::UNIT == A_TILE_BYTES + FmtNvfp4::SFA && FmtMxfp8::UNIT == A_TILE_BYTES + FmtMxfp8::SFA,
              "activation unit = codes + scales");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;            // 256 FP32 columns
constexpr uint32_t SF_COL = 256;           // scale factors, one column set per ring stage:
constexpr uint32_t SF_STAGE_COLS = 48;     //   A: 4 K-groups x 4 columns, then B: 4 K-groups x 8
constexpr uint32_t SFB_OFF = 16;
constexpr int kMaxStages = 5;
// Two ring shapes, one K step per stage (measured against two K steps per stage, whose
// operands arrive in fewer, larger copies: 2.21 vs 1.99-2.04 ms at prefill16k, the coarser
// ring leaves the MMA waiting longer).
//   Full (A holds 128 rows, 4 stages): the weight tile (B codes, B scales), then at the next
//     1 KB boundary the activation unit (A codes, A scales): a K step of a 128-row block is
//     two copies, one per operand (each copy has a fixed cost in the SM's copy path).  A
//     block of fewer rows copies A's codes and scales of its rows only, as two copies.
//   Small-M (batches of <= 32 tokens, so every expert has <= 32 rows; 5 stages): A holds 32
//     rows and comes first, A | B | SFB | SFA, which leaves room for a 5th stage of weights in
//     flight.  The MMA still reads 128 rows of A; rows past the region read the stage's own B
//     bytes and only feed accumulator rows that are never stored.  A's codes and scales are
//     two copies of only the rows present.
// Offsets are 1 KB aligned where the swizzled operands start.
template <int kStages, int kABytes, class F = FmtNvfp4>
struct Ring {
  using Fmt = F;
  static constexpr int STAGES = kStages;
  static constexpr int A_BYTES = kABytes;
  static constexpr bool kFullA = kABytes == A_TILE_BYTES;
  static constexpr int OFF_B = kFullA ? 0 : kABytes;  // B codes, then B scales
  static constexpr int OFF_A = kFullA ? (F::TILE + 1023) / 1024 * 1024 : 0;
  static constexpr int OFF_SFA = kFullA ? OFF_A + kABytes : kABytes + F::TILE;
  static constexpr int STAGE_BYTES = (OFF_SFA + F::SFA + 1023) / 1024 * 1024;
  static_assert(SF_COL + kStages * SF_STAGE_COLS <= TMEM_COLS, "scale-factor stages must fit in TMEM");
  static_assert(kStages <= kMaxStages, "barrier arrays");
};
using RingFull = Ring<4, A_TILE_BYTES>;
using RingSmallM = Ring<5, 32 * BK_BYTES>;
using RingFullMx = Ring<4, A_TILE_BYTES, FmtMxfp8>;
using RingSmallMMx = Ring<5, 32 * BK_BYTES, FmtMxfp8>;
static_assert(RingFull::STAGE_BYTES == A_TILE_BYTES + kTileBytes + SFA_BYTES, "NVFP4 stages need no padding");
constexpr int NUM_EPI_WARPS = 16;
constexpr int NUM_SF_WARPS = 4;                      // one per TMEM lane quarter
constexpr int FIRST_SF_WARP = 2 + NUM_EPI_WARPS;
constexpr int NUM_THREADS = (2 + NUM_EPI_WARPS + NUM_SF_WARPS) * 32;
constexpr int kEpiGroups = NUM_EPI_WARPS / 4;  // column groups: each warp owns a lane quarter x group
static_assert(kEpiGroups * 64 == BN && kEpiGroups * 32 * 2 == BN, "down: 64 columns, gate/up: 32 + 32 per group");
constexpr int kTileSlots = 4;       // tile ids the producer may publish ahead of the epilogue

// Instruction descriptor: E2M1 A and B (format 1), E4M3 scales (format 0), K-major
// operands, N = 256 (n_dim = N/8 at bit 17), M = 128 (m_dim = M/16 at bit 24).
constexpr uint32_t kIdescNvfp4 = (1u << 7) | (1u << 10) | ((BN >> 3) << 17) | ((BM >> 4) << 24);
// E4M3 A and B (format 0), UE8M0 scales (bit 23), K-major, N = 256, M = 128.  The scale
// byte of MMA kb within each 32-bit TMEM scale cell is selected by the A and B
// scale-factor ids (bits 29-30 and 4-5).
constexpr uint32_t kIdescMxf8 = (1u << 23) | ((BN >> 3) << 17) | ((BM >> 4) << 24);
__host__ __device__ constexpr uint32_t idesc_mxf8(int kb) {
  return kIdescMxf8 | (static_cast<uint32_t>(kb) << 29) | (static_cast<uint32_t>(kb) << 4);
}

struct __align__(16) GemmSmemTail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tile_full[kTileSlots];   // producer -> MMA + epilogue: tile id published
  uint64_t tile_empty[kTileSlots];  // MMA + epilogue + scale warps -> producer: slot read
  uint64_t sf_full[kMaxStages];     // scale warps -> MMA: stage's scale factors are in TMEM
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  int tile_ids[kTileSlots];         // claimed tile, -1 = no more work
  int4 tile_mb[kTileSlots][2];      // its block-list entry (MBlock), read once by the producer
  uint32_t tmem_base;
  int abort_flag;
};

template <class R>
static size_t ring_smem_bytes() {
  return static_cast<size_t>(R::STAGES) * R::STAGE_BYTES + sizeof(GemmSmemTail) + 1024;
}

// silu(g) * u in FP32 with the fast exponential and division (a few ulp; h is compared with
// the FP64 oracle within its tolerance, unlike the quantiser steps, which stay exact).  For
// g -> -inf, exp(-g) = inf and g / inf = -0.
__device__ __forceinline__ float silu_times(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }


__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Waits until *counter >= target (acquire at GPU scope, or at system scope for counters
// that other GPUs add to).  Returns false (and sets *abort) when the wait ran past
// kWaitLimitNs or another role already aborted.
template <bool kSys = false>
__device__ __forceinline__ bool wait_counter_bounded(const uint32_t* counter, uint32_t target,
                                                     volatile int* abort_flag) {
  auto load = [&]() { return kSys ? ld_acquire_sys(counter) : ld_acquire_gpu(counter); };
  if (load() >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(64);
    if (load() >= target) return true;
    if ((i & 15u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Block-list entries are written by the routing kernels; read them from L2.
__device__ __forceinline__ MBlock load_mblock(const MBlock* p) {
  const int4 v = __ldcg(reinterpret_cast<const int4*>(p));
  const int4 u = __ldcg(reinterpret_cast<const int4*>(p) + 1);
  return MBlock{v.x, v.y, v.z, v.w, __int_as_float(u.x), __int_as_float(u.y), {0, 0}};
}

// Position of a tile id in the list [gate/up tiles of every block][down tiles of every block].
struct TileRef {
  bool down;
  int block;  // index into the block list
  int nt;     // 256-column output tile
};

__device__ __forceinline__ TileRef tile_ref(int id, int total_gu, int n_gu, int n_d) {
  TileRef t;
  t.down = id >= total_gu;
  const int rel = t.down ? id - total_gu : id;
  const int n = t.down ? n_d : n_gu;
  t.block = rel / n;
  t.nt = rel - t.block * n;
  return t;
}

template <class R>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_experts_kernel(const ExpertGemmArgs args) {
  constexpr int STAGES = R::STAGES, A_BYTES = R::A_BYTES, STAGE_BYTES = R::STAGE_BYTES;
  using F = typename R::Fmt;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GemmSmemTail* tail = reinterpret_cast<GemmSmemTail*>(smem + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &tail->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
      mbar_init(&tail->sf_full[s], NUM_SF_WARPS);
    }
    for (int j = 0; j < kTileSlots; ++j) {
      mbar_init(&tail->tile_full[j], 1);
      mbar_init(&tail->tile_empty[j], 1 + NUM_EPI_WARPS + NUM_SF_WARPS);
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
  // The block list and the zeroed scheduler words come from the routing kernels, two or
  // more launches back, which are complete once this grid runs (every kernel of the forward
  // triggers its dependents only after its own wait).  Only the activations A1 come from the
  // previous kernel, so the producer claims tiles and streams the first stages' weights
  // before it waits; every other thread waits here.
  const bool producer = warp == 0 && lane == 0;
  if (!producer) {
    pdl_wait();
    pdl_trigger();
  }

  const int n_gu = args.gu_n_tiles, n_d = args.d_n_tiles;
  const int num_blocks = __ldcg(args.num_mblocks);
  const int total_gu = num_blocks * n_gu;
  const int total = total_gu + num_blocks * n_d;
  uint32_t* const ready = args.sched + 1;
  const uint32_t ready_target = static_cast<uint32_t>(n_gu) * NUM_EPI_WARPS;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, slot = 0;
      uint32_t phase = 0, slot_phase = 0;
      uint32_t armed = 0, armed_parity = 0;
      // The next claim is issued while the current tile's last STAGES K steps are still to
      // be loaded, so its round trip hides behind them instead of opening a gap in the ring.
      uint32_t claim = atomicAdd(args.sched, 1u);
      bool waited = false;  // grid dependency resolved: activations may be read
      for (;;) {
        if (!mbar_wait_bounded(&tail->tile_empty[slot], slot_phase ^ 1, abort_flag)) break;
        int id = claim < static_cast<uint32_t>(total) ? static_cast<int>(claim) : -1;
        // the tile's block entry travels with its id, so no consumer reads global memory for it
        const TileRef t = tile_ref(id < 0 ? 0 : id, total_gu, n_gu, n_d);
        const MBlock mb = id < 0 ? MBlock{} : load_mblock(args.mblocks + t.block);
        tail->tile_ids[slot] = id;
        tail->tile_mb[slot][0] = make_int4(mb.expert, mb.row_begin, mb.rows, mb.sf_block);
        tail->tile_mb[slot][1] = make_int4(__float_as_int(mb.scale_gu), __float_as_int(mb.scale_d), 0, 0);
        mbar_arrive(&tail->tile_full[slot]);
        if (++slot == kTileSlots) {
          slot = 0;
          slot_phase ^= 1;
        }
        if (id < 0) break;
        const int k_tiles = t.down ? args.d_k_tiles : args.gu_k_tiles;
        const int n_tiles = t.down ? n_d : n_gu;
        const uint8_t* a_src = (t.down ? args.a2 : args.a1) + static_cast<size_t>(mb.sf_block) * k_tiles * F::UNIT;
        const uint8_t* btile = (t.down ? args.w_d : args.w_gu) +
                               (static_cast<size_t>(mb.expert) * n_tiles + t.nt) * k_tiles * static_cast<size_t>(F::TILE);
        if (t.down) {
          // this block's A2 is written by the gate/up epilogues (possibly of other CTAs)
          if (!wait_counter_bounded(ready + t.block, ready_target, abort_flag)) {
            atomicOr(args.err, kErrTimeoutProducer);
            break;
          }
          fence_proxy_async_global();
        } else if (args.arrivals) {
          // expert parallelism: this block's A1 rows are stored by the ranks that route them
          if (!wait_counter_bounded<true>(args.arrivals + t.block, static_cast<uint32_t>(mb.rows), abort_flag)) {
            atomicOr(args.err, kErrTimeoutProducer);
            break;
          }
          fence_proxy_async_global();
        }
        // A block of 128 rows in the full ring: the whole unit, one copy.  Otherwise the
        // codes and the scales of the block's valid rows (rounded up to 8; the MXFP8 atom
        // holds all rows' scales), two copies: the stale shared-memory rows past them only
        // reach accumulator rows never stored.
        uint32_t a_bytes = static_cast<uint32_t>(min(BM, (mb.rows + 7) & ~7)) * BK_BYTES;
        if (a_bytes > static_cast<uint32_t>(A_BYTES)) {  // cannot happen when the host picks the ring right
          atomicOr(args.err, kErrRange);
          a_bytes = A_BYTES;
        }
        const bool whole = R::kFullA && a_bytes == static_cast<uint32_t>(A_TILE_BYTES);
        const uint32_t sfa_bytes = F::kMx ? F::SFA : a_bytes / 8;  // NVFP4: 16 scale bytes per row
        const uint32_t a_copy = whole ? F::UNIT : a_bytes + sfa_bytes;
        // A and its scales of K step kk into stage st
        auto load_a = [&](int st, int kk) {
          uint8_t* sp = smem + st * STAGE_BYTES;
          const uint8_t* unit = a_src + static_cast<size_t>(kk) * F::UNIT;
          if (whole) {
            bulk_load(sp + R::OFF_A, unit, F::UNIT, &tail->full[st]);
          } else {
            bulk_load(sp + R::OFF_A, unit, a_bytes, &tail->full[st]);
            bulk_load(sp + R::OFF_SFA, unit + A_TILE_BYTES, sfa_bytes, &tail->full[st]);
          }
        };
        // Before the wait only the weights are loaded; the first tile starts at stage 0, so
        // its deferred K steps kk < STAGES sit in stages kk.
        int deferred = 0;
        auto resolve = [&]() {
          pdl_wait();
          pdl_trigger();
          waited = true;
          for (int kk = 0; kk < deferred; ++kk) load_a(kk, kk);
        };
        bool ok = true;
        const int claim_at = max(0, k_tiles - STAGES);
        for (int kt = 0; kt < k_tiles; ++kt) {
          if (kt == claim_at) claim = atomicAdd(args.sched, 1u);
          if (!waited && kt == STAGES) resolve();
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&tail->full[stage], a_copy + F::TILE);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          bulk_load(smem + stage * STAGE_BYTES + R::OFF_B, btile + static_cast<size_t>(kt) * F::TILE, F::TILE,
                    &tail->full[stage]);
          if (waited)
            load_a(stage, kt);
          else
            ++deferred;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!waited) resolve();
        if (!ok) break;
      }
      if (!waited) {  // no tile claimed
        pdl_wait();
        pdl_trigger();
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
      int stage = 0, slot = 0;
      uint32_t phase = 0, acc_phase = 0, slot_phase = 0;
      for (;;) {
        if (!mbar_wait_bounded(&tail->tile_full[slot], slot_phase, abort_flag)) break;
        const int id = tail->tile_ids[slot];
        mbar_arrive(&tail->tile_empty[slot]);
        if (++slot == kTileSlots) {
          slot = 0;
          slot_phase ^= 1;
        }
        if (id < 0) break;
        const int k_tiles = id >= total_gu ? args.d_k_tiles : args.gu_k_tiles;
        if (!mbar_wait_bounded(&tail->acc_empty, acc_phase ^ 1, abort_flag)) break;
        tc_fence_after();
        bool ok = true;
        for (int kt = 0; kt < k_tiles; ++kt) {
          // the stage's operands have landed and its scale factors are in TMEM
          if (!mbar_wait_bounded(&tail->sf_full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES + R::OFF_A);
          const uint32_t sb = smem_u32(smem + stage * STAGE_BYTES + R::OFF_B);
          const uint32_t sf = tmem + SF_COL + stage * SF_STAGE_COLS;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            if constexpr (F::kMx)  // the 4 MMAs share the stage's scale columns, byte kb of each cell
              tc_mma_mxf8(tmem + ACC_COL, sdesc_k_sw128(sa + kb * 32), sdesc_k_sw128(sb + kb * 32), idesc_mxf8(kb),
                          sf, sf + SFB_OFF, (kt | kb) != 0 ? 1u : 0u);
            else
              tc_mma_nvfp4(tmem + ACC_COL, sdesc_k_sw128(sa + kb * 32), sdesc_k_sw128(sb + kb * 32), kIdescNvfp4,
                           sf + kb * 4, sf + SFB_OFF + kb * 8, (kt | kb) != 0 ? 1u : 0u);
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
  } else if (warp >= FIRST_SF_WARP) {
    // ------------------------------------------------------------ scale factors -> TMEM
    // Each warp fills its own lane quarter of the stage's scale-factor columns: per K-group,
    // lane l writes the 4 scales of rows l, l + 32, l + 64, l + 96 into 4 columns (B: from
    // the weight tile's 512-byte atoms, which hold them in that order; NVFP4 A: gathered
    // from the stage's [128 rows][16 scales]), every quarter getting the same columns, so
    // the MMA finds the scales of row m at lane m, column + m / 32.  Doing it
    // with tcgen05.st keeps these copies off the tensor pipe, which then only runs MMAs.
    const int quarter = warp & 3;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int stage = 0, slot = 0;
    uint32_t phase = 0, slot_phase = 0;
    for (;;) {
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tail->tile_full[slot], slot_phase, abort_flag))) break;
      const int id = tail->tile_ids[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tile_empty[slot]);
      if (++slot == kTileSlots) {
        slot = 0;
        slot_phase ^= 1;
      }
      if (id < 0) break;
      const int k_tiles = id >= total_gu ? args.d_k_tiles : args.gu_k_tiles;
      bool ok = true;
      for (int kt = 0; kt < k_tiles; ++kt) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tail->full[stage], phase, abort_flag))) {
          ok = false;
          break;
        }
        const uint8_t* ssfb = smem + stage * STAGE_BYTES + R::OFF_B + B_BYTES;  // [half][K-group][512]
        const uint8_t* ssfa = smem + stage * STAGE_BYTES + R::OFF_SFA;  // NVFP4 [128 rows][16]; MXFP8 one atom
        const uint32_t col = SF_COL + stage * SF_STAGE_COLS;
        if constexpr (F::kMx) {
          // one atom of A scales -> columns 0..3; B: rows 0-127 -> SFB_OFF + 0..3, rows 128-255 -> + 4..7
          const uint4 a = *reinterpret_cast<const uint4*>(ssfa + lane * 16);
          const uint32_t ra[4] = {a.x, a.y, a.z, a.w};
          tmem_st_32x32b_x4(t_lane + col, ra);
          const uint4 b0 = *reinterpret_cast<const uint4*>(ssfb + lane * 16);
          const uint4 b1 = *reinterpret_cast<const uint4*>(ssfb + 512 + lane * 16);
          const uint32_t rb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          tmem_st_32x32b_x8(t_lane + col + SFB_OFF, rb);
        } else {
          uint32_t r[16];
          // A: the stage holds [128 rows][16 scales]; K-group kb -> columns 4 kb .. 4 kb + 3,
          // column 4 kb + q of lane l = the 4 scales of row l + 32 q in that K-group
          {
            const uint4 q0 = *reinterpret_cast<const uint4*>(ssfa + lane * 16);
            const uint4 q1 = *reinterpret_cast<const uint4*>(ssfa + (lane + 32) * 16);
            const uint4 q2 = *reinterpret_cast<const uint4*>(ssfa + (lane + 64) * 16);
            const uint4 q3 = *reinterpret_cast<const uint4*>(ssfa + (lane + 96) * 16);
            r[0] = q0.x; r[1] = q1.x; r[2] = q2.x; r[3] = q3.x;
            r[4] = q0.y; r[5] = q1.y; r[6] = q2.y; r[7] = q3.y;
            r[8] = q0.z; r[9] = q1.z; r[10] = q2.z; r[11] = q3.z;
            r[12] = q0.w; r[13] = q1.w; r[14] = q2.w; r[15] = q3.w;
          }
          tmem_st_32x32b_x16(t_lane + col, r);
          // B: K-group kb -> columns 8 kb .. 8 kb + 3 (rows 0-127), 8 kb + 4 .. 8 kb + 7 (rows 128-255)
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int kb = part * 2 + q;
              const uint4 v0 = *reinterpret_cast<const uint4*>(ssfb + kb * 512 + lane * 16);
              const uint4 v1 = *reinterpret_cast<const uint4*>(ssfb + SFB_BYTES / 2 + kb * 512 + lane * 16);
              r[q * 8 + 0] = v0.x; r[q * 8 + 1] = v0.y; r[q * 8 + 2] = v0.z; r[q * 8 + 3] = v0.w;
              r[q * 8 + 4] = v1.x; r[q * 8 + 5] = v1.y; r[q * 8 + 6] = v1.z; r[q * 8 + 7] = v1.w;
            }
            tmem_st_32x32b_x16(t_lane + col + SFB_OFF + part * 16, r);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tail->sf_full[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;            // TMEM lanes this warp may access
    const int group = (warp - 2) >> 2;       // column group: gate/up 32 + 32 columns, down 64
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float alpha2 = args.alpha_a2;
    const float six_alpha2 = __fmul_rn(6.0f, alpha2);
    int slot = 0;
    uint32_t acc_phase = 0, slot_phase = 0;
    for (;;) {
      // every lane waits; the warp leaves together if any lane gave up, so the warp-wide
      // operations below never run with part of the warp gone
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tail->tile_full[slot], slot_phase, abort_flag))) break;
      const int id = tail->tile_ids[slot];
      const int4 m0 = tail->tile_mb[slot][0], m1 = tail->tile_mb[slot][1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tile_empty[slot]);
      if (++slot == kTileSlots) {
        slot = 0;
        slot_phase ^= 1;
      }
      if (id < 0) break;
      const TileRef t = tile_ref(id, total_gu, n_gu, n_d);
      const MBlock mb{m0.x, m0.y, m0.z, m0.w, __int_as_float(m1.x), __int_as_float(m1.y), {0, 0}};
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tail->acc_full, acc_phase, abort_flag))) break;
      tc_fence_after();
      uint32_t v[2][32];
      if (!t.down) {  // gate columns [group*32, +32) and the matching up columns
        tmem_ld_32x32b_x32(t_lane + ACC_COL + group * 32, v[0]);
        tmem_ld_32x32b_x32(t_lane + ACC_COL + 128 + group * 32, v[1]);
      } else {
        tmem_ld_32x32b_x32(t_lane + ACC_COL + group * 64, v[0]);
        tmem_ld_32x32b_x32(t_lane + ACC_COL + group * 64 + 32, v[1]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->acc_empty);
      acc_phase ^= 1;
      const bool valid = row_in_tile < mb.rows;
      if (!t.down) {
        if (valid && F::kMx) {
          // 32 features = one MX block: 32 E4M3 codes (chunks c, c + 1 of K tile f0 / 128)
          // and one scale byte (block f0 / 32 of the row: byte f0 / 32 % 4 of its K tile's word)
          const float scale = mb.scale_gu;
          const int f0 = t.nt * 128 + group * 32;
          float h[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            h[i] = silu_times(__uint_as_float(v[0][i]) * scale, __uint_as_float(v[1][i]) * scale);
          uint32_t c[8];
          const uint32_t sc = quant_block32_mx(h, c);
          st_act_pair(args.a2, mb.sf_block, args.d_k_tiles, f0 >> 7, row_in_tile, (f0 & 127) >> 4, c);
          args.a2[sf_atom_offset(mb.sf_block, args.d_k_tiles, row_in_tile, f0 >> 5)] = static_cast<uint8_t>(sc);
        } else if (valid) {
          const float scale = mb.scale_gu;
          const int f0 = t.nt * 128 + group * 32;  // first feature of this thread's 32
          uint32_t codes[4];
          uint32_t scodes = 0;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float h[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g = __uint_as_float(v[0][b * 16 + i]) * scale;
              const float u = __uint_as_float(v[1][b * 16 + i]) * scale;
              h[i] = silu_times(g, u);
            }
            const uint32_t sc = quant_block16(h, alpha2, six_alpha2, codes[2 * b], codes[2 * b + 1]);
            scodes |= sc << (8 * b);
          }
          // 32 features = one 16-byte chunk (f0 % 256) / 32 of K tile f0 / 256 of the A2 tile
          *reinterpret_cast<uint4*>(args.a2 + act_tile_offset(mb.sf_block, args.d_k_tiles, f0 >> 8, row_in_tile,
                                                              (f0 & 255) >> 5)) =
              make_uint4(codes[0], codes[1], codes[2], codes[3]);
          // its 2 scales are 2 contiguous bytes of the row's 16 in its K step (f0 / 16 is even)
          *reinterpret_cast<uint16_t*>(args.a2 + sf_chunk_offset(mb.sf_block, args.d_k_tiles, row_in_tile,
                                                                    f0 / 16)) = static_cast<uint16_t>(scodes);
        }
        // publish this warp's share of block t.block's A2 to the down-tile producers
        fence_proxy_async_global();
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          atomicAdd(ready + t.block, 1u);
        }
      } else if (valid) {
        const float scale = mb.scale_d;
        const size_t r = static_cast<size_t>(mb.row_begin + row_in_tile);
        // 64 BF16 = 128 contiguous bytes of row r, written as 4 x 32-byte stores
        uint16_t* dst = args.y + r * args.y_cols + t.nt * BN + group * 64;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t p[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = q * 16 + 2 * i;
            p[i] = bf16x2_bits(__uint_as_float(v[c >> 5][c & 31]) * scale,
                               __uint_as_float(v[(c + 1) >> 5][(c + 1) & 31]) * scale);
          }
          st_global_v8(dst + q * 16, p);
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

template <class R>
static cudaError_t launch_ring(const ExpertGemmArgs& a, int grid, cudaStream_t s) {
  const size_t smem = ring_smem_bytes<R>();
  cudaError_t e = cudaFuncSetAttribute(gemm_experts_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_experts_kernel<R>, dim3(grid), dim3(NUM_THREADS), smem, s, a);
}

cudaError_t launch_gemm_experts(const ExpertGemmArgs& a, int grid, cudaStream_t s) {
  // With at most 32 tokens no expert has more than 32 rows.
  if (a.max_rows_per_expert <= 32) return launch_ring<RingSmallM>(a, grid, s);
  return launch_ring<RingFull>(a, grid, s);
}

cudaError_t launch_gemm_experts_mx(const ExpertGemmArgs& a, int grid, cudaStream_t s) {
  if (a.max_rows_per_expert <= 32) return launch_ring<RingSmallMMx>(a, grid, s);
  return launch_ring<RingFullMx>(a, grid, s);
}

}  // namespace beam
