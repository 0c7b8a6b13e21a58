// Device helpers shared by the kernels of libbeam_moe: error word, bounded waits, PTX
// wrappers for mbarrier / TMA / tcgen05 (sm_100a), and the NVFP4 / BF16 conversions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace beam {

// ---------------------------------------------------------------- device error word
// Bits set by kernels; beam_moe_check reads and clears them.
enum : uint32_t {
  kErrTimeoutProducer = 1u << 0,
  kErrTimeoutMma = 1u << 1,
  kErrTimeoutEpilogue = 1u << 2,
  kErrRange = 1u << 8,
};

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialisation may start while the previous
// kernel in the stream is still running.  pdl_wait() blocks until that kernel has finished
// and its memory is visible (a no-op for a normal launch); every kernel of the forward
// calls it before touching memory that another kernel of the stream writes or reads.
// pdl_trigger() lets the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with parity `parity` of `bar`.  Returns false (and sets *abort)
// when the wait ran past kWaitLimitNs or another role already aborted.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Orders this thread's generic-proxy global accesses with its later async-proxy (bulk
// copy) accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// The same for shared memory of this CTA.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// The same at system scope: words that other GPUs write (peer stores over NVLink).
__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void red_add_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("red.release.sys.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// CTA arrival: release of this CTA's stores (ordered before it by the barrier) and acquire
// of every earlier arrival's, at GPU scope (all CTAs of the grid share the GPU).
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------- TMA / bulk copies
// 2-D tiled TMA load (no multicast) completing on `bar` with complete_tx bytes.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Contiguous bulk copy global -> shared (addresses 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Asks L2 to fetch a contiguous range (16-byte aligned, bytes % 16 == 0); no completion.
__device__ __forceinline__ void prefetch_l2(const void* gsrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}
// Same for one box of a 2-D tensor map.
__device__ __forceinline__ void prefetch_l2_tile(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrives once on `bar` when every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// Shared memory -> TMEM: 32 rows of 16 bytes, broadcast to the four 32-lane quarters.
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// D(tmem) (+)= A(smem) * B(smem)^T, NVFP4 operands with E4M3 block-16 scales in TMEM.
__device__ __forceinline__ void tc_mma_nvfp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// D(tmem) (+)= A(smem) * B(smem)^T, E4M3 operands (K = 32 per MMA) with one UE8M0 scale
// per 32 values in TMEM; the scale byte within each 32-bit TMEM cell comes from the
// instruction descriptor's scale-factor ids.
__device__ __forceinline__ void tc_mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// D(tmem) (+)= A(smem) * B(smem)^T, BF16 operands, FP32 accumulation.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Registers -> TMEM: lane i of the warp writes N consecutive 32-bit columns of TMEM lane
// (taddr lane + i), starting at taddr's column (the warp's own lane quarter only).
__device__ __forceinline__ void tmem_st_32x32b_x4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
               "r"(r[2]), "r"(r[3])
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, K-major operand with the 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), layout type 2.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);  // start address
  d |= static_cast<uint64_t>(1u) << 16;                // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;        // stride byte offset
  d |= static_cast<uint64_t>(1u) << 46;                // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                // 128-byte swizzle
  return d;
}
// Same for the 64-byte swizzle: rows of 64 bytes, 8-row groups 512 bytes apart, type 4.
__device__ __forceinline__ uint64_t sdesc_k_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(512u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(4u) << 61;
  return d;
}
// Descriptor of a 32-row x 16-byte source for tcgen05.cp: 8-row core matrices of
// contiguous 16-byte rows, 128 bytes apart, no swizzle.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(0u) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

// ---------------------------------------------------------------- number formats
// Two FP32 -> packed E2M1 byte (lo in the low nibble), round-to-nearest-even, saturating.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}
// FP32 (finite, >= 0) -> E4M3 code, round-to-nearest-even, saturating to 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}
// Unsigned E4M3 code -> exact FP32 value (codes produced here are never NaN).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * (1.0f / 512.0f);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// NVFP4 quantisation of one block of 16 FP32 values with tensor scale alpha:
// s = amax / (6 alpha), S = E4M3(s), d = S alpha, q_i = E2M1(v_i / d); S == 0 -> all 0
// (every step an IEEE FP32 operation).
// Writes 8 code bytes (little-endian in two uint32) and returns the scale code.
__device__ __forceinline__ uint32_t quant_block16(const float (&v)[16], float alpha, float six_alpha, uint32_t& lo,
                                                  uint32_t& hi) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sc = cvt_e4m3(__fdiv_rn(amax, six_alpha));
  if (sc == 0) {
    lo = hi = 0;
    return 0;
  }
  const float d = __fmul_rn(e4m3_value(sc), alpha);
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = cvt_e2m1x2(__fdiv_rn(v[2 * i], d), __fdiv_rn(v[2 * i + 1], d));
  lo = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  hi = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
  return sc;
}

// ---------------------------------------------------------------- MXFP8
// Two FP32 -> two signed E4M3 codes in the low 16 bits (lo in the low byte),
// round-to-nearest-even, saturating to +-448, sign of zero kept.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Scale exponent of an MX block: the smallest e with amax <= 448 * 2^e, clamped below at
// -127.  With amax = m * 2^E, m in [1, 2): 448 = 1.75 * 2^8, so e = E - 8 when m <= 1.75
// (mantissa bits <= 0x600000), else E - 7.  Zero and subnormal amax give -127.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = static_cast<int>((b >> 23) & 0xFFu);
  if (ef == 0) return -127;
  const int e = ef - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : e;
}

// MXFP8 of one block of 32 FP32 values: scale X = 2^e (mx_scale_exp of the block's amax),
// codes E4M3(v_i / X).  v_i * 2^-e is exact (a power-of-two scaling that stays normal, or
// falls below 2^-126 where it encodes to zero either way).  Writes the 32 code bytes as 8
// little-endian words and returns the UE8M0 scale code e + 127.
__device__ __forceinline__ uint32_t quant_block32_mx(const float (&v)[32], uint32_t (&c)[8]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx_scale_exp(amax);
  // 2^-e as an FP32: e in [-127, 120], so -e + 127 is a normal biased exponent in [7, 254]
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t p0 = cvt_e4m3x2(__fmul_rn(v[4 * i], inv), __fmul_rn(v[4 * i + 1], inv));
    const uint32_t p1 = cvt_e4m3x2(__fmul_rn(v[4 * i + 2], inv), __fmul_rn(v[4 * i + 3], inv));
    c[i] = p0 | (p1 << 16);
  }
  return static_cast<uint32_t>(e + 127);
}

// Activation units.  The expert inputs (A1) and the SwiGLU outputs (A2) of each 128-row
// block are stored K step by K step, one unit per K step: first the step's codes, a tile of
// 128 rows x 128 bytes (NVFP4: 256 values, MXFP8: 128), row m at m * 128 and its 16-byte
// chunk c at ((c ^ (m % 8)) * 16) (the 128-byte swizzle the tensor core reads), then the
// step's scales (NVFP4: [128 rows][16] bytes; MXFP8: one 512-byte atom).  A K step of the
// activations and its scales are therefore one contiguous copy for the GEMM.
constexpr int kActCodeBytes = 16384;
constexpr int kActUnitNvfp4 = kActCodeBytes + 128 * 16;
constexpr int kActUnitMx = kActCodeBytes + 512;

// NVFP4: byte offset of 16-byte code chunk c of row m in K step kt of `block`.
__device__ __forceinline__ size_t act_tile_offset(size_t block, int k_tiles, int kt, int m, int c) {
  return (block * static_cast<size_t>(k_tiles) + static_cast<size_t>(kt)) * kActUnitNvfp4 +
         static_cast<size_t>(m * 128 + ((c ^ (m & 7)) << 4));
}

// One 32-byte store (8 x 32 bits) to a 32-byte aligned global address.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// MXFP8: 32 code bytes = 16-byte chunks c and c + 1 (c even) of row m in K step kt of
// `block`.  Under the swizzle the two chunks fill one 32-byte aligned span
// (c ^ (m % 8) and (c + 1) ^ (m % 8) differ only in bit 0), chunk c first when m is even
// and second when m is odd; one 32-byte store writes both.
__device__ __forceinline__ void st_act_pair(uint8_t* tiles, size_t block, int k_tiles, int kt, int m, int c,
                                            const uint32_t (&w)[8]) {
  uint8_t* p = tiles + (block * static_cast<size_t>(k_tiles) + static_cast<size_t>(kt)) * kActUnitMx +
               static_cast<size_t>(m * 128 + ((c ^ (m & 6)) << 4));
  const bool swap = (m & 1) != 0;
  uint32_t s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) s[i] = swap ? w[(i + 4) & 7] : w[i];
  st_global_v8(p, s);
}

// NVFP4 activation scales: the 16 scales of one K step (256 values) of the 128 rows of a
// block follow the step's codes as a [128 rows][16] chunk, row m's 16 bytes at m * 16, so a
// row's scales of a K step are one contiguous store for the writers.  (The 512-byte-atom
// order of the tensor cores scattered a row's scales in 4-byte pieces 512 bytes apart, whose
// partial-sector writes held the A1 writer at ~3.4 TB/s where 16-byte pieces reach ~4.5 TB/s;
// the GEMM's scale warps gather the atom order from the chunk.)  Byte offset of scale s of
// row m of `block`, in the same buffer as the codes:
__device__ __forceinline__ size_t sf_chunk_offset(size_t block, int k_tiles, int m, int s) {
  return (block * static_cast<size_t>(k_tiles) + static_cast<size_t>(s >> 4)) * kActUnitNvfp4 + kActCodeBytes +
         static_cast<size_t>(m * 16 + (s & 15));
}

// MXFP8 activation scales: scale s of row m (0..127) of `block` (K/128 K steps of four
// scales) in the 512-byte atom after its K step's codes (the tcgen05 scale-factor atom order).
__device__ __forceinline__ size_t sf_atom_offset(size_t block, int k_tiles, int m, int s) {
  return (block * static_cast<size_t>(k_tiles) + static_cast<size_t>(s >> 2)) * kActUnitMx + kActCodeBytes +
         static_cast<size_t>((m & 31) * 16 + (m >> 5) * 4 + (s & 3));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Exclusive prefix sum of one int per thread over the whole CTA (blockDim.x <= 1024, a
// multiple of 32); *total gets the sum.  warp_sums: 33 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) warp_sums[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? warp_sums[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += u;
    }
    if (lane < nwarps) warp_sums[lane] = si - s;  // exclusive prefix of warp totals
    if (lane == 31) warp_sums[32] = si;           // grand total
  }
  __syncthreads();
  total = warp_sums[32];
  const int r = warp_sums[warp] + inc - v;
  __syncthreads();
  return r;
}

}  // namespace beam
