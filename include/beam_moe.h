/*
 * beam_moe.h — C ABI of libbeam_moe.so: the forward pass of one Beam-style sparse
 * mixture-of-experts layer on one NVIDIA B200 (sm_100a).
 *
 * The layer (sources are web pages, cited by title and section):
 *   - router GEMM from hidden 5120 to 256 expert logits, computed in FP32
 *     (vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Status": router GEMM
 *     kernels for (5120, 256); news article "vLLM adds day-zero Reflection Beam serving",
 *     section "Agents worked on the serving path": a specialised FP32 router kernel);
 *   - softmax over all experts, the top 8 of 256 (vLLM recipe
 *     "reflection/Beam-1.0-501B-A23B", section "Overview"), weights renormalised over
 *     the chosen 8;
 *   - routed experts in NVFP4, W4A4 on Blackwell (recipe, section "Variants"), SwiGLU;
 *     or, as the second precision variant, block-scaled FP8 W8A8 experts (the recipe's FP8
 *     checkpoint, same section), read as MXFP8 (beam_moe_create_mxfp8);
 *   - MoE finalize: weighted un-permute, post-RMSNorm of the sandwich norm (eps 1e-6)
 *     and residual add (PR, sections "Status" and "Remaining work").
 *
 * Conventions for every entry point:
 *   - Pointers are device pointers unless the name says _host.  `stream` is a
 *     cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - Work is enqueued asynchronously on `stream`; nothing synchronises the host except
 *     beam_moe_create, beam_moe_check and beam_moe_destroy, which say so.
 *   - Errors are returned as a beam_moe_status and never thrown.  Argument errors are
 *     found on the host before anything is enqueued.  Faults found on the device (a wait
 *     that ran out of time, an index out of range) set a device error word that
 *     beam_moe_check reports.
 *   - BF16 tensors are passed as raw 16-bit patterns (uint16_t / void*).
 *   - Activation and weight tensors must start on a 16-byte boundary (the kernels use
 *     16-byte vector accesses); a misaligned pointer is rejected with INVALID_ARG.
 *   - NVFP4 data: two 4-bit E2M1 codes per byte, element 2i in the low nibble; one
 *     unsigned E4M3 scale byte per 16 consecutive elements of a row; one FP32 tensor
 *     scale alpha per tensor; value = e2m1 * e4m3 * alpha.
 *   - MXFP8 data (the block-scaled FP8 expert variant, beam_moe_create_mxfp8): one
 *     signed E4M3 code per byte; one UE8M0 scale byte S per 32 consecutive elements of a
 *     row (an exponent with bias 127); no tensor scale; value = e4m3 * 2^(S - 127).
 */
#ifndef BEAM_MOE_H_
#define BEAM_MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BEAM_MOE_API __attribute__((visibility("default")))
#else
#define BEAM_MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BEAM_MOE_OK = 0,
  BEAM_MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, tokens > max_tokens ...  */
  BEAM_MOE_ERR_UNSUPPORTED = 2, /* a shape this build does not handle (see create)      */
  BEAM_MOE_ERR_CUDA = 3,        /* a CUDA runtime call failed                           */
  BEAM_MOE_ERR_OOM = 4,         /* device allocation failed                              */
  BEAM_MOE_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (reported by check)    */
  BEAM_MOE_ERR_DEVICE = 6       /* a device-side range check failed (reported by check) */
} beam_moe_status;

/* Layer shape and the static activation scales.  Supported: hidden % 256 == 0,
 * inter % 128 == 0, 1 <= top_k <= 16, top_k <= num_experts <= 1024,
 * num_experts % 32 == 0 or num_experts < 32, max_tokens >= 1. */
typedef struct {
  int32_t max_tokens;  /* largest num_tokens a forward may be called with              */
  int32_t hidden;      /* H (5120)                                                    */
  int32_t num_experts; /* E (256)                                                     */
  int32_t top_k;       /* k (8)                                                       */
  int32_t inter;       /* I, expert intermediate size                                 */
  float rms_eps;       /* post-RMSNorm epsilon (1e-6)                                 */
  float alpha_a1;      /* FP32 tensor scale of the NVFP4 expert inputs (> 0)          */
  float alpha_a2;      /* FP32 tensor scale of the NVFP4 SwiGLU outputs (> 0)         */
} beam_moe_config;

/* Layer weights (device pointers, read only during beam_moe_create; the caller keeps
 * ownership and may free them after create returns). */
typedef struct {
  const float* router_w;     /* [E][H] FP32, row e = expert e                           */
  const uint8_t* w_gu;       /* [E][2I][H/2] NVFP4 codes; rows 0..I-1 gate, I..2I-1 up  */
  const uint8_t* w_gu_sf;    /* [E][2I][H/16] E4M3 scales, row-major                     */
  const float* w_gu_alpha;   /* [E] tensor scale of each expert's gate+up                */
  const uint8_t* w_d;        /* [E][H][I/2] NVFP4 codes of the down projection          */
  const uint8_t* w_d_sf;     /* [E][H][I/16] E4M3 scales                                 */
  const float* w_d_alpha;    /* [E] tensor scale of each expert's down                   */
  const uint16_t* gamma;     /* [H] BF16 RMSNorm weight                                  */
} beam_moe_weights;

typedef struct beam_moe_ctx* beam_moe_t;

/* Validates cfg, allocates the handle's device memory (repacked weights and a workspace
 * sized for cfg->max_tokens), repacks the weights into the tensor-core layout on `stream`
 * and synchronises `stream` before returning.  On success *out owns all of it until
 * beam_moe_destroy.  Returns INVALID_ARG / UNSUPPORTED / OOM / CUDA. */
BEAM_MOE_API beam_moe_status beam_moe_create(const beam_moe_config* cfg, const beam_moe_weights* weights, void* stream,
                                beam_moe_t* out);

/* Block-scaled FP8 (W8A8) experts, the second precision variant of the routed experts
 * (recipe "reflection/Beam-1.0-501B-A23B", section "Variants": an FP8 checkpoint next to
 * the NVFP4 one).  The pages do not give the FP8 block layout; this library reads it as
 * the OCP microscaling format MXFP8, which the sm_100a tensor cores scale natively:
 * E4M3 values, one power-of-two scale per 32 values along the contraction dimension,
 * for the weights and for both activations (A1 = MX(x), A2 = MX(SwiGLU)).  Activation
 * scales are chosen per 32-value block on the device: 2^e with e the smallest integer
 * such that amax <= 448 * 2^e (e >= -127), so nothing saturates. */
typedef struct {
  const float* router_w;   /* [E][H] FP32, row e = expert e                              */
  const uint8_t* w_gu;     /* [E][2I][H] E4M3 codes; rows 0..I-1 gate, I..2I-1 up       */
  const uint8_t* w_gu_sf;  /* [E][2I][H/32] UE8M0 scales, row-major                     */
  const uint8_t* w_d;      /* [E][H][I] E4M3 codes of the down projection              */
  const uint8_t* w_d_sf;   /* [E][H][I/32] UE8M0 scales                                 */
  const uint16_t* gamma;   /* [H] BF16 RMSNorm weight                                    */
} beam_moe_weights_mxfp8;

/* beam_moe_create for MXFP8 experts.  cfg->alpha_a1 and cfg->alpha_a2 are not used (MX
 * activations have no tensor scale).  Same shape limits, ownership, synchronisation and
 * errors as beam_moe_create.  Every other entry point takes the handle unchanged. */
BEAM_MOE_API beam_moe_status beam_moe_create_mxfp8(const beam_moe_config* cfg, const beam_moe_weights_mxfp8* weights,
                                                   void* stream, beam_moe_t* out);

/* Expert format of a handle: BEAM_MOE_FMT_NVFP4 or BEAM_MOE_FMT_MXFP8 (-1 for NULL). */
enum { BEAM_MOE_FMT_NVFP4 = 0, BEAM_MOE_FMT_MXFP8 = 1 };
BEAM_MOE_API int32_t beam_moe_expert_format(beam_moe_t h);

/* out[T][H] = residual + RMSNorm(sum_j w_j * expert_{id_j}(x)) * gamma, rounded to BF16.
 * x, residual, out: [num_tokens][H] BF16 row-major, caller-owned, device memory.
 * out may equal residual (in-place residual update); no other aliasing.  0 <= num_tokens
 * <= max_tokens (0 enqueues nothing).  Uses the handle's workspace, so calls on one
 * handle must be ordered (same stream, or synchronised). */
BEAM_MOE_API beam_moe_status beam_moe_forward(beam_moe_t h, const void* x, const void* residual, void* out, int32_t num_tokens,
                                 void* stream);

/* beam_moe_forward fused with the next sublayer's sandwich pre-norm (the PR's sandwich
 * norms fused with the MoE finalize): besides out, writes
 *   next_x[T][H] = bf16( out / sqrt(mean(out^2) + next_eps) * next_gamma ),
 * computed from the BF16 out values.  next_gamma: [H] BF16 device pointer (the next
 * sublayer's pre-norm weight); next_x must not alias x, residual or out.  Same errors as
 * beam_moe_forward. */
BEAM_MOE_API beam_moe_status beam_moe_forward_prenorm(beam_moe_t h, const void* x, const void* residual, void* out,
                                                      void* next_x, const void* next_gamma, float next_eps,
                                                      int32_t num_tokens, void* stream);

/* Same as beam_moe_forward with HOST buffers: copies x to the handle's device staging
 * buffer on `stream`, runs the forward, copies out back on `stream`; the residual's copy
 * starts once x has landed and runs on a second stream of the handle, overlapping the
 * routing and the expert GEMMs; only the finalize waits for it (the first call creates that
 * stream and two events).
 * Batches of 2 x BEAM_MOE_HOST_CHUNK_TOKENS tokens or more (beam_moe_set_host_chunk_tokens)
 * run in parts of that many tokens: the second stream uploads each part's x and residual in
 * turn, `stream` runs each part's forward as its x lands, and a third stream of the handle
 * copies each part's out back as soon as it is final, under the later parts' uploads.  The
 * parts take the whole batch's router, finalize and GEMM forms, so out has the same bits as
 * without parts.  Not with BEAM_MOE_ROUTER_SIMT.  After such a call the internal buffers
 * (beam_moe_debug_copy) and the kernel timings hold the last part's.
 * An out of at most 2 MB in page-locked memory that the device can address (cudaHostAlloc,
 * or registered with cudaHostRegisterMapped) is written by the finalize kernel directly, with
 * no copy after it; larger outs and other host memory go through a staging buffer and a
 * copy back.
 * All copies are cudaMemcpyAsync; pinned host memory makes them asynchronous.  The work
 * enqueued on `stream` ends with out_host complete: the caller synchronises `stream` before
 * reading it. */
BEAM_MOE_API beam_moe_status beam_moe_forward_host(beam_moe_t h, const void* x_host, const void* residual_host, void* out_host,
                                      int32_t num_tokens, void* stream);

/* ---- Tensor parallelism over the experts' intermediate size, with the finalize fused to
 * its all-reduce (vLLM PR "Day-0 support for Reflection's Beam-1.0", section "Status":
 * Beam's TP all-reduce fused with the sandwich norms and the MoE finalize; recipe
 * "reflection/Beam-1.0-501B-A23B": NVFP4 with TP4 on Blackwell).
 *
 * Each of W ranks (one process per GPU) creates an ordinary handle (beam_moe_create or
 * beam_moe_create_mxfp8) from its slice of the experts: cfg->inter = I / W, the gate rows
 * and the up rows of features [r I/W, (r+1) I/W) and the same columns of the down weights
 * (the tensor scales of the whole tensors unchanged; I / W must meet create's limits).
 * Router weights and gamma are the full ones on every rank.  Then, once per group:
 *   1. beam_moe_tp_region: the handle allocates its exchange region (device memory it owns:
 *      a flag header, two [max_tokens][H] FP32 buffers and one [max_tokens][H] BF16 buffer)
 *      and returns its address;
 *   2. the ranks exchange the regions (beam_moe_ipc_export / beam_moe_ipc_import across
 *      processes, or plain pointers when the ranks share a process and a GPU);
 *   3. beam_moe_tp_attach with every rank's region, in rank order.
 * beam_moe_forward_tp then computes out on every rank (identical bits on all ranks): the
 * routing, A1 and the expert GEMMs of the rank's slice, its partial m, the exchange, and
 * the post-RMSNorm + residual of the summed m.  Below 256 tokens the all-reduce is one-shot
 * (every rank reads all W partials of every token); from 256 tokens on it is two-shot: rank r
 * reduces and finishes only tokens [r S, (r + 1) S), S = ceil(T / W), publishes those BF16
 * rows in its region, and then copies the other ranks' rows into out (T H 4 + T H 2 bytes
 * read per rank instead of W T H 4).  Both forms give the same bits.  Every rank must call it
 * the same number of times, with the same num_tokens, like a collective.  A rank that waits
 * more than 2 s for its peers gives up: beam_moe_check then returns BEAM_MOE_ERR_TIMEOUT. */
#define BEAM_MOE_IPC_HANDLE_BYTES 64
BEAM_MOE_API int64_t beam_moe_tp_region_bytes(beam_moe_t h);
/* Allocates the region on the first call (synchronises the device); *region gets its
 * device address (256-byte aligned). */
BEAM_MOE_API beam_moe_status beam_moe_tp_region(beam_moe_t h, void** region);
/* regions: host array of `world` device addresses (regions[rank] must be this handle's own
 * region); 1 <= world <= 16.  Synchronises `stream` and the device, clears this rank's
 * flags.  Call on every rank before the group's first forward. */
BEAM_MOE_API beam_moe_status beam_moe_tp_attach(beam_moe_t h, int32_t rank, int32_t world, void* const* regions,
                                                void* stream);
/* x, residual, out, num_tokens as beam_moe_forward (out on every rank; out may equal
 * residual).  Enqueued on `stream`; the exchange waits on the device, not the host. */
BEAM_MOE_API beam_moe_status beam_moe_forward_tp(beam_moe_t h, const void* x, const void* residual, void* out,
                                                 int32_t num_tokens, void* stream);
/* beam_moe_forward_tp in three parts: phase 0 = routing, GEMMs, this rank's partial m and
 * its publication; phase 1 = the wait for every rank's partials, their sum, norm and residual
 * (of every token, or of this rank's slice in the two-shot form, then published); phase 2 =
 * the two-shot form's wait for every rank's rows and their copy into out (nothing is
 * enqueued in the one-shot form).  Phases run in order (0, 1, 2, 0, ...) with the same
 * num_tokens; phase 1 and 2 need residual and out.  Splitting lets ranks that share one GPU
 * run every rank's phase p before any phase p + 1, so no kernel waits on a kernel that has
 * not run. */
BEAM_MOE_API beam_moe_status beam_moe_forward_tp_phase(beam_moe_t h, const void* x, const void* residual, void* out,
                                                       int32_t num_tokens, int32_t phase, void* stream);
/* The batch size from which beam_moe_forward_tp reduces in two steps (default
 * BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS; INT32_MAX keeps the one-shot form for every batch).  A
 * batch whose slices would not all hold a token (T < W^2 can do that) stays one-shot.  Both
 * forms give the same bits; the choice only moves the exchange's bytes and latency.  Takes
 * effect at the next phase 0; all ranks of a group must use the same value.  Not from the
 * source pages: exposed for tuning and testing.  INVALID_ARG for min_tokens < 1. */
#define BEAM_MOE_TP_TWO_SHOT_MIN_TOKENS 256
BEAM_MOE_API beam_moe_status beam_moe_set_tp_two_shot_tokens(beam_moe_t h, int32_t min_tokens);
/* Part size of beam_moe_forward_host (tokens, a multiple of 256, the router's largest token
 * tile; default BEAM_MOE_HOST_CHUNK_TOKENS; 0 = a batch is never split).  Parts of 4096
 * tokens keep each part's expert GEMMs compute-bound (every part reads the weights of the
 * experts it routes to) while the host copies, 4 H bytes per token, set the pace.  Not from
 * the source pages: an implementation choice exposed for tuning and testing.  INVALID_ARG
 * for tokens < 0 or not a multiple of 256. */
#define BEAM_MOE_HOST_CHUNK_TOKENS 4096
BEAM_MOE_API beam_moe_status beam_moe_set_host_chunk_tokens(beam_moe_t h, int32_t tokens);
/* cudaIpcGetMemHandle / cudaIpcOpenMemHandle / cudaIpcCloseMemHandle of a region, as
 * BEAM_MOE_IPC_HANDLE_BYTES opaque bytes (host memory), so that callers need no CUDA
 * headers. */
BEAM_MOE_API beam_moe_status beam_moe_ipc_export(const void* dev_ptr, void* handle_out);
BEAM_MOE_API beam_moe_status beam_moe_ipc_import(const void* handle, void** dev_ptr);
BEAM_MOE_API beam_moe_status beam_moe_ipc_close(void* dev_ptr);

/* ---- Expert parallelism with attention data parallelism (vLLM PR "Day-0 support for
 * Reflection's Beam-1.0", section "Status": Attention DP with the MegaMoE kernels; recipe,
 * "Overview": 8 of 256 experts; "Launching the server": expert parallel with data-parallel
 * attention).  Each of W ranks holds experts [expert_begin, expert_begin + expert_count)
 * with expert_begin = rank * expert_count and expert_count * W = E (cfg->num_experts = all
 * E, used for routing; the weight arrays and the tensor scales hold only the rank's
 * experts, in order) and its own batch of num_tokens tokens, the same num_tokens on every
 * rank; cfg->max_tokens bounds W * num_tokens.  Only routed rows travel.
 * beam_moe_forward_ep, in four phases:
 *   0  route the rank's own tokens; publish its per-expert row counts to every rank;
 *   1  wait for every rank's counts and derive the common layout (each rank's received rows,
 *      expert-major, within an expert by source rank then token); quantise each own token
 *      once and store each slot's row into the activation tiles of its expert's rank (peer
 *      stores), adding it to that block's arrival count;
 *   2  the expert GEMMs over the rows this rank received (a block's gate/up tiles start as
 *      soon as all its rows have arrived), then every output row back to its source slot
 *      (peer stores) and a return flag;
 *   3  wait for every rank's return flag; finalize the rank's own tokens from the returned
 *      rows (slot order, this rank's routing weights).
 * Each token's output is bit-identical to the single-GPU forward of the same tokens.
 * Regions, exchange and attach as for tensor parallelism (beam_moe_tp_region /
 * beam_moe_ipc_* / beam_moe_tp_attach; attach checks the expert ranges);
 * beam_moe_forward and beam_moe_forward_tp refuse these handles (INVALID_ARG).  A rank that
 * waits more than 2 s for its peers gives up: beam_moe_check then returns TIMEOUT. */
BEAM_MOE_API beam_moe_status beam_moe_create_ep(const beam_moe_config* cfg, const beam_moe_weights* weights,
                                                int32_t expert_begin, int32_t expert_count, void* stream,
                                                beam_moe_t* out);
BEAM_MOE_API beam_moe_status beam_moe_create_ep_mxfp8(const beam_moe_config* cfg, const beam_moe_weights_mxfp8* weights,
                                                      int32_t expert_begin, int32_t expert_count, void* stream,
                                                      beam_moe_t* out);
/* x, residual, out: this rank's [num_tokens][H] BF16 (device).  Like a collective: every
 * rank calls it the same number of times with the same num_tokens. */
BEAM_MOE_API beam_moe_status beam_moe_forward_ep(beam_moe_t h, const void* x, const void* residual, void* out,
                                                 int32_t num_tokens, void* stream);
/* One phase (0, 1, 2, 3, in turn, the same num_tokens) of beam_moe_forward_ep, so that ranks
 * sharing one GPU can run every rank's phase p before any rank's phase p + 1; any other
 * order returns INVALID_ARG. */
BEAM_MOE_API beam_moe_status beam_moe_forward_ep_phase(beam_moe_t h, const void* x, const void* residual, void* out,
                                                       int32_t num_tokens, int32_t phase, void* stream);

/* Bytes of logits_ws that beam_moe_route needs for this shape (the logits may be held as
 * partial sums over slices of H).  0 for empty shapes. */
BEAM_MOE_API int64_t beam_moe_route_workspace_bytes(int32_t num_tokens, int32_t hidden, int32_t num_experts);

/* Routing alone, on caller buffers: logits[T][E] = x W_r^T (FP32 arithmetic), then the
 * top-k of the softmax (ties: lower expert index) in descending weight and the weights
 * renormalised over the chosen k.  x [T][H] BF16, router_w [E][H] FP32; logits_ws is
 * caller scratch of beam_moe_route_workspace_bytes(T, H, E) bytes; ids [T][k] int32 and
 * w [T][k] FP32 are outputs.  Same shape limits as beam_moe_config. */
BEAM_MOE_API beam_moe_status beam_moe_route(const void* x, const float* router_w, int32_t num_tokens, int32_t hidden,
                               int32_t num_experts, int32_t top_k, float* logits_ws, int32_t* ids, float* w,
                               void* stream);

/* Routing without any device allocation.  The pages have no counterpart of this entry
 * point: it exists for callers that cannot call cudaMalloc, such as plugins inside a host
 * engine that owns all device memory and hands them only their inputs and outputs, or
 * latency-critical loops where an allocation (and the device synchronisation it can
 * imply) is not allowed after start-up.  Same result as beam_moe_route (same kernels),
 * but the logits scratch is a fixed 8 MiB array compiled into this library: every GPU
 * that loads the library holds it until the process exits.
 *   - Accepts exactly the shapes whose logits fit the array: S(T, H, E) * T * E <= 2^21
 *     floats, where S is the number of slices of H the router sums (the rule of
 *     beam_moe_route_workspace_bytes(T, H, E) <= 8 MiB).  S falls as T grows (8, 4, 2, 1
 *     at H = 5120, E = 256), so the accepted T are not one interval: at H = 5120,
 *     E = 256 they are 1..1024, 1153..2048, 2305..4096 and 4673..8192.  Other shapes
 *     return BEAM_MOE_ERR_UNSUPPORTED before anything is enqueued.
 *   - The first call on each device looks up the array's device address (with that
 *     device current) and caches it; make that first call before any stream capture.
 *     The address is looked up again only when the device's CUDA context has changed
 *     (a device reset): the first call after such a change should also come before any
 *     stream capture.
 *   - All calls on a device share the one array, which keeps the last call's contents
 *     (every element a call reads it first writes, so nothing needs clearing).  Calls
 *     that overlap on the GPU (different streams, or different host threads) race on it:
 *     order them.
 *   - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 * Arguments and outputs as beam_moe_route, without logits_ws. */
BEAM_MOE_API beam_moe_status beam_moe_route_static(const void* x, const float* router_w, int32_t num_tokens,
                                                   int32_t hidden, int32_t num_experts, int32_t top_k, int32_t* ids,
                                                   float* w, void* stream);

/* NVFP4 quantiser Q (weights or activations): src [rows][cols] FP32 row-major, cols %
 * 16 == 0.  codes [rows][cols/2], sf [rows][cols/16] (row-major scale bytes).  alpha >
 * 0 uses that tensor scale; alpha <= 0 computes alpha = amax(src) / 2688 on the device
 * first.  If alpha_out is not NULL the scale used is written there (device FP32). */
BEAM_MOE_API beam_moe_status beam_moe_quantize_nvfp4(const float* src, int64_t rows, int64_t cols, float alpha, uint8_t* codes,
                                        uint8_t* sf, float* alpha_out, void* stream);

/* MXFP8 quantiser (weights or activations), the rule of beam_moe_create_mxfp8:
 * src [rows][cols] FP32 row-major, finite, cols % 32 == 0.  codes [rows][cols] E4M3,
 * sf [rows][cols/32] UE8M0 (row-major scale bytes).  codes must be 16-byte aligned. */
BEAM_MOE_API beam_moe_status beam_moe_quantize_mxfp8(const float* src, int64_t rows, int64_t cols, uint8_t* codes,
                                                     uint8_t* sf, void* stream);

/* Internal buffers of the last forward, for tests (layouts in the comment of each id). */
typedef enum {
  BEAM_MOE_BUF_LOGITS = 0,   /* [S][T][E] FP32 partial sums over S slices of H (S = size/(4TE)) */
  BEAM_MOE_BUF_IDS = 1,      /* [T][k] int32                                               */
  BEAM_MOE_BUF_WEIGHTS = 2,  /* [T][k] FP32                                                */
  BEAM_MOE_BUF_OFFSETS = 3,  /* [E+1] int32: rows of expert e are [off[e], off[e+1])       */
  BEAM_MOE_BUF_PERM = 4,     /* [T*k] int32: token of permuted row r                        */
  BEAM_MOE_BUF_INV = 5,      /* [T][k] int32: permuted row of (token, slot)                */
  BEAM_MOE_BUF_SFBLOCK = 6,  /* [E+1] int32: first 128-row scale block of each expert      */
  BEAM_MOE_BUF_A1 = 7,       /* activation units (below) of the permuted expert inputs, K = H */
  BEAM_MOE_BUF_A2 = 8,       /* activation units of the SwiGLU outputs, K = Ip = ceil(I/256)*256 */
  BEAM_MOE_BUF_Y = 9         /* [T*k][H] BF16 expert outputs in permuted row order          */
} beam_moe_buffer;
/* Blocks: the rows of expert e, local row i = r - off[e], live in block
 * blk = sfblock[e] + i/128, row m = i%128.
 * Activation units: one per block and K step of 256 values, U = 18432 bytes, the step's
 * 16384 code bytes (128 rows x 128) followed by its 2048 scale bytes (128 rows x 16), so
 * the expert GEMM loads a K step of codes and scales with one copy.  In unit
 * u = blk * (K/256) + j/128, code byte j of that row (values 2j, 2j+1) is at
 * u*U + m*128 + ((((j%128)/16) ^ (m%8)) * 16) + j%16, and scale s (values 16s .. 16s+15),
 * in unit blk * (K/256) + s/16, at u*U + 16384 + m*16 + s%16.
 * MXFP8 handles: one value per code byte, one scale per 32 values, K steps of 128 values
 * and U = 16896 (16384 code bytes, then a 512-byte scale atom in the tensor cores'
 * scale-factor order): code j (value j) in unit u = blk * (K/128) + j/128 at
 * u*U + m*128 + ((((j%128)/16) ^ (m%8)) * 16) + j%16, scale s in unit blk * (K/128) + s/4
 * at u*U + 16384 + (m%32)*16 + (m/32)*4 + s%4, and A2's K is I (no padding). */

/* Copies min(bytes, size of the buffer) bytes of internal buffer `which` to dst (device),
 * enqueued on `stream`.  *size_out (host, may be NULL) receives the buffer's size for the
 * last forward's num_tokens. */
BEAM_MOE_API beam_moe_status beam_moe_debug_copy(beam_moe_t h, int32_t which, void* dst, size_t bytes, size_t* size_out,
                                    void* stream);

/* Synchronises `stream`, then reads and clears the device error word.  Returns OK,
 * TIMEOUT or DEVICE. */
BEAM_MOE_API beam_moe_status beam_moe_check(beam_moe_t h, void* stream);

/* Router for batches of more than 16 tokens (16 or fewer use the fused small-batch routing
 * kernel).  SIMT: FP32 FFMA over slices of H, then a top-k kernel that sums the slices.
 * TENSOR: the tensor cores on the exact three-part BF16 split of the FP32 weights, over
 * (128-token tiles) x (slices of H) with partial logits summed by the top-k kernel (about
 * one wave of CTAs below 4096 tokens, two from there); once a single slice fills two waves
 * (about 37,900 tokens on 148 SMs), one 256-token tile per CTA with the top-k in its
 * epilogue.  AUTO (the default) is TENSOR from BEAM_MOE_ROUTER_TC_SPLIT_MIN_TOKENS tokens
 * on.  All compute FP32-accurate logits and differ only in the order of the FP32 additions.
 * Not from the source pages: an implementation choice exposed for testing and tuning.
 * Returns INVALID_ARG for an unknown mode. */
enum { BEAM_MOE_ROUTER_AUTO = 0, BEAM_MOE_ROUTER_SIMT = 1, BEAM_MOE_ROUTER_TENSOR = 2 };
#define BEAM_MOE_ROUTER_TC_SPLIT_MIN_TOKENS 17
BEAM_MOE_API beam_moe_status beam_moe_set_router_mode(beam_moe_t h, int32_t mode);

/* Per-kernel timing.  While enabled (enable != 0), beam_moe_forward records a CUDA event
 * on `stream` before its first kernel and after each kernel it enqueues.  Creating the
 * events is the only allocation; enable once, outside any timed region. */
BEAM_MOE_API beam_moe_status beam_moe_profile_enable(beam_moe_t h, int32_t enable);

/* Waits for the events of the last profiled forward and writes the duration in ms of each
 * of its kernels, in launch order, to ms[0 .. min(capacity, count)); *count (host) gets
 * the number of kernels.  Names of the kernels: beam_moe_kernel_name. */
BEAM_MOE_API beam_moe_status beam_moe_profile_read(beam_moe_t h, float* ms, int32_t capacity, int32_t* count);

/* Name of the index-th kernel of the last forward ("router", "topk", ...), or NULL. */
BEAM_MOE_API const char* beam_moe_kernel_name(beam_moe_t h, int32_t index);

/* Failure-detection check: enqueues one CTA that waits, with the same bounded mbarrier
 * wait as the GEMM kernels, on a barrier nothing completes.  After limit_ns (1 ns .. 2 s)
 * it gives up, sets the timeout bit of the device error word and exits normally, so the
 * next beam_moe_check returns BEAM_MOE_ERR_TIMEOUT and the context stays usable. */
BEAM_MOE_API beam_moe_status beam_moe_debug_wait_timeout(beam_moe_t h, int64_t limit_ns, void* stream);

/* Number of kernels the last beam_moe_forward enqueued. */
BEAM_MOE_API int32_t beam_moe_last_launch_count(beam_moe_t h);

BEAM_MOE_API const char* beam_moe_status_string(beam_moe_status s);

/* Synchronises the device, then frees everything the handle owns.  NULL is a no-op. */
BEAM_MOE_API void beam_moe_destroy(beam_moe_t h);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H_ */
