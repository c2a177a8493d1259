/*
 * beam_moe.h - C ABI of the B200 (sm_100a) Beam MoE block forward.
 *
 * The operation is the routed-expert block of the Beam model as the Hugging
 * Face launch post "Welcome Beam" describes it in section "Mixture of
 * Experts": every expert is scored with a sigmoid of the router logits, the
 * experts are split into n_group groups, the topk_group groups with the best
 * sum of their two top scores are kept, the top_k experts inside them are
 * chosen, each chosen expert is a SwiGLU MLP, and the expert outputs are
 * combined with normalized router weights scaled by routed_scale (2.5 in
 * Beam). Section "Residual Stream" of the same post fixes the router and the
 * SwiGLU product to FP32; this library computes the router logits, the
 * sigmoid, the selection, the weights and the SwiGLU product in FP32, the
 * expert matmuls as BF16 x BF16 with FP32 accumulation.
 *
 * Conventions shared by every entry point:
 *  - Pointers named as device buffers must be device memory of the current
 *    device; the caller owns all of them and the library never frees them.
 *    All row-major. bf16 is passed as its 16-bit pattern (uint16_t).
 *  - Every pointer must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *    default stream); nothing synchronizes except beam_moe_check and
 *    beam_moe_trace_read.
 *  - Host-side checks run before any launch; on any error nothing is
 *    launched and the outputs are untouched.
 *  - T = 0 is a no-op that returns BEAM_MOE_OK.
 *  - Results are bitwise reproducible run to run (no atomics on data).
 *  - The library allocates no device memory: scratch lives in the caller's
 *    workspace `ws` (size from beam_moe_workspace_size). A workspace must not
 *    be shared by calls that may run concurrently.
 */
#ifndef BEAM_MOE_H
#define BEAM_MOE_H

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

/* Block configuration. Beam: {5120, 2560, 256, 8, 4, 8, 1, 0, 2.5f, 0}.
 * Supported: hidden and inter multiples of 128; n_experts <= 512 and a
 * multiple of n_group; group size (n_experts / n_group) >= 2; top_k <= 32 and
 * top_k <= topk_group * group size; see beam_moe_status for the codes. */
typedef struct beam_moe_cfg {
  int32_t hidden;      /* H: model width                                   */
  int32_t inter;       /* I: expert intermediate width                     */
  int32_t n_experts;   /* E: routed experts                                */
  int32_t n_group;     /* G: expert groups (E / G experts each)            */
  int32_t topk_group;  /* Gk: groups kept per token                        */
  int32_t top_k;       /* K: experts per token                             */
  int32_t renormalize; /* 1: w_k = S s_k / sum_j s_j; 0: w_k = S s_k       */
  int32_t bias_mode;   /* 0: bias added to the logits before the sigmoid;
                          1: bias added to the scores for choosing only,
                             weights from the unbiased scores (DeepSeek-V3) */
  float routed_scale;  /* S: multiplies the combined output (2.5 in Beam)  */
  int32_t router_tc;   /* 0 (default): the FP32 router GEMM is a chain of
                          FP32 FMAs on CUDA cores. 1 (opt-in): the same
                          contraction on tensor cores, each FP32 router
                          weight split exactly into three bf16 parts whose
                          products with the bf16 x are exact, summed by the
                          tensor core's FP32 accumulator (its rounding of
                          the sums is not an FMA chain's; about 6x faster
                          for large batches). Needs hidden % 64 == 0,
                          else the CUDA-core kernel runs.                  */
} beam_moe_cfg;

typedef enum beam_moe_status {
  BEAM_MOE_OK = 0,
  BEAM_MOE_ERR_INVALID_ARG = 1,       /* NULL / negative / inconsistent argument   */
  BEAM_MOE_ERR_UNSUPPORTED_SHAPE = 2, /* configuration outside the supported set  */
  BEAM_MOE_ERR_ALIGNMENT = 3,         /* a pointer is not 16-byte aligned         */
  BEAM_MOE_ERR_WORKSPACE_TOO_SMALL = 4,
  BEAM_MOE_ERR_CUDA = 5,              /* a CUDA runtime/driver call failed        */
  BEAM_MOE_ERR_DEVICE_TIMEOUT = 6     /* a kernel gave up a bounded wait          */
} beam_moe_status;

typedef enum beam_moe_op {
  BEAM_MOE_OP_ROUTE = 0,         /* beam_moe_route                            */
  BEAM_MOE_OP_FORWARD = 1,       /* beam_moe_forward, beam_moe_forward_routed */
  BEAM_MOE_OP_FORWARD_NVFP4 = 2, /* beam_moe_forward_nvfp4                    */
  BEAM_MOE_OP_FORWARD_HOST = 3,  /* beam_moe_forward_host                      */
  BEAM_MOE_OP_FORWARD_NVFP4_HOST = 4, /* beam_moe_forward_nvfp4_host          */
} beam_moe_op;

/* Bytes of workspace the operation needs for T tokens (a pure host function). */
BEAM_MOE_API beam_moe_status beam_moe_workspace_size(const beam_moe_cfg* cfg, int64_t T, beam_moe_op op,
                                        size_t* bytes);

/*
 * Router and selection ("Welcome Beam", section "Mixture of Experts": sigmoid
 * scores, groups ranked by the sum of their top two scores, top experts inside
 * the kept groups, normalized weights).
 *   x          [T][H] bf16, device            token activations
 *   w_router   [E][H] fp32, device            router weights
 *   bias       [E] fp32, device, or NULL      per-expert bias (see bias_mode)
 *   topk_ids   [T][K] int32, device (out)     chosen experts, by descending
 *                                             choice score, ties to lower id
 *   topk_w     [T][K] fp32, device (out)      combine weights, S included
 *   expert_counts [E] int32, device, or NULL (out): tokens routed to each expert
 *   ws, ws_bytes  device workspace of at least
 *                 beam_moe_workspace_size(cfg, T, BEAM_MOE_OP_ROUTE) bytes
 */
BEAM_MOE_API beam_moe_status beam_moe_route(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                               const float* w_router, const float* bias, int32_t* topk_ids,
                               float* topk_w, int32_t* expert_counts, void* ws, size_t ws_bytes,
                               void* stream);

/*
 * Routing without any device allocation and without a caller workspace. No
 * page describes such a call: this entry point exists for callers that cannot
 * call cudaMalloc, for example a serving process whose memory pool has already
 * reserved the GPU's memory for weights and caches, or a runtime that forbids
 * device allocations once it has started. The caller still passes inputs and
 * outputs exactly as for beam_moe_route (same meaning, layout and alignment);
 * the scratch is a fixed BEAM_MOE_NOALLOC_SCRATCH_BYTES array inside the
 * library, which every GPU that loads the library holds until the process
 * exits.
 *  - Limits: T <= BEAM_MOE_NOALLOC_MAX_TOKENS and n_experts <=
 *    BEAM_MOE_NOALLOC_MAX_EXPERTS; larger calls return
 *    BEAM_MOE_ERR_WORKSPACE_TOO_SMALL before anything is launched.
 *  - The first call on a device looks up the array's device address for that
 *    device (once, with that device current); make that first call before
 *    any stream capture on the device. The address is kept for the life of
 *    the process, so a device reset (cudaDeviceReset, or a reset of the
 *    primary context) after the first call is not supported.
 *  - Every call on a device shares the one array: calls that may overlap on
 *    the GPU (different streams, no ordering between them) race and must be
 *    serialized by the caller.
 *  - Results equal beam_moe_route's up to the order of FP32 partial sums of
 *    the router logits (the number of H splits may differ).
 */
#define BEAM_MOE_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
#define BEAM_MOE_NOALLOC_MAX_TOKENS 2048
#define BEAM_MOE_NOALLOC_MAX_EXPERTS 256
BEAM_MOE_API beam_moe_status beam_moe_route_noalloc(const beam_moe_cfg* cfg, int64_t T,
                                                    const uint16_t* x, const float* w_router,
                                                    const float* bias, int32_t* topk_ids,
                                                    float* topk_w, int32_t* expert_counts,
                                                    void* stream);

/*
 * Whole block forward: routing as beam_moe_route, then for every token
 *   out[t] = sum_k topk_w[t][k] * Wd_e (silu(Wg_e x_t) * (Wu_e x_t)),  e = topk_ids[t][k]
 * ("Welcome Beam", section "Mixture of Experts": SwiGLU experts of
 * intermediate size I, outputs combined with normalized weights and scaled).
 *   w13  [E][2I][H] bf16, device   rows 0..I-1 gate (Wg), rows I..2I-1 up (Wu)
 *   w2   [E][H][I]  bf16, device   down projection (Wd)
 *   out  [T][H]     bf16, device (out)
 *   topk_ids, topk_w, expert_counts: optional device outputs (NULL to skip)
 *   ws, ws_bytes: at least beam_moe_workspace_size(cfg, T, BEAM_MOE_OP_FORWARD)
 */
BEAM_MOE_API beam_moe_status beam_moe_forward(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                 const float* w_router, const float* bias, const uint16_t* w13,
                                 const uint16_t* w2, uint16_t* out, int32_t* topk_ids,
                                 float* topk_w, int32_t* expert_counts, void* ws,
                                 size_t ws_bytes, void* stream);

/*
 * Expert path with caller-supplied routes (routing replay, as the Miles
 * "Beam 1.0" page's rollout routing replay option reuses recorded routes):
 * the same as beam_moe_forward after its routing step.
 *   topk_ids [T][K] int32, device: distinct experts per token, each in [0, E)
 *   topk_w   [T][K] fp32, device: combine weights (any scale already applied)
 * Ids are not re-validated on the device beyond a bounds check that flags
 * BEAM_MOE_ERR_DEVICE_TIMEOUT-class status bit 0x100 in beam_moe_check.
 */
BEAM_MOE_API beam_moe_status beam_moe_forward_routed(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                        const int32_t* topk_ids, const float* topk_w,
                                        const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                                        int32_t* expert_counts, void* ws, size_t ws_bytes,
                                        void* stream);

/*
 * NVFP4 experts ("Welcome Beam", section "Mixture of Experts": the NVFP4
 * checkpoint stores most parameters in 4-bit precision for NVIDIA Blackwell
 * GPUs). A value is e2m1(code) * e4m3(scale) * tensor_scale: 4-bit E2M1 codes
 * {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit, packed two per byte (element
 * 2j in the low nibble), one FP8 E4M3 scale per 16 consecutive elements of a
 * row, one FP32 scale per tensor. Scales are stored in the block-scaled MMA
 * layout: for a matrix with K elements per row, the scale of row r and
 * 16-element block b is at byte
 *   ((r / 128) * (K / 64) + b / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + b % 4.
 * All pointers are device memory, 16-byte aligned.
 */
typedef struct beam_moe_nvfp4_experts {
  const uint8_t* w13_codes;  /* [E][2I][H/2]: rows 0..I-1 gate, I..2I-1 up   */
  const uint8_t* w13_scales; /* E * 2I * H / 16 bytes, layout above (K = H)  */
  const uint8_t* w2_codes;   /* [E][H][I/2]                                  */
  const uint8_t* w2_scales;  /* E * H * I / 16 bytes, layout above (K = I)   */
  float w13_scale;           /* tensor scale of W13                          */
  float w2_scale;            /* tensor scale of W2                           */
  float x_scale;             /* tensor scale x is quantised with             */
  float h_scale;             /* tensor scale h = silu(g) * u is quantised with */
} beam_moe_nvfp4_experts;

/*
 * Whole block with NVFP4 experts and NVFP4 activations (W4A4, the scheme of
 * the vLLM recipe's FlashInfer TRT-LLM NVFP4 backend): routing as
 * beam_moe_forward; every token's x is quantised per 16 elements (scale =
 * e4m3(amax / (6 x_scale)), code = e2m1(x / (scale x_scale)), round to
 * nearest even, saturating); g, u = W13 x on block-scaled FP4 tensor cores
 * with FP32 accumulation; h = silu(g) * u in FP32, quantised the same way with
 * h_scale; y = W2 h in FP32; out as beam_moe_forward. Requires hidden and
 * inter to be multiples of 256. Workspace: BEAM_MOE_OP_FORWARD_NVFP4.
 */
BEAM_MOE_API beam_moe_status beam_moe_forward_nvfp4(const beam_moe_cfg* cfg, int64_t T,
                                                    const uint16_t* x, const float* w_router,
                                                    const float* bias,
                                                    const beam_moe_nvfp4_experts* experts,
                                                    uint16_t* out, int32_t* topk_ids,
                                                    float* topk_w, int32_t* expert_counts,
                                                    void* ws, size_t ws_bytes, void* stream);

/*
 * The block forward on activations in HOST memory, the call a serving loop
 * makes with a batch it holds on the host. x_host [T][H] bf16 and out_host
 * [T][H] bf16 are host buffers (page-locked, or the copies cannot overlap);
 * w_router, bias, w13, w2 and ws are device memory as for beam_moe_forward.
 * The result equals beam_moe_forward's for the same tokens. Batches of at
 * least 2 * BEAM_MOE_HOST_CHUNK tokens run in chunks of that many tokens
 * (bf16 batches of at least 8 * BEAM_MOE_HOST_CHUNK in chunks twice that
 * size, so that each chunk's GEMMs stay compute-bound): the host-to-device
 * copy of chunk i + 1 and the device-to-host copy of chunk i - 1 run on two
 * copy streams the call creates, while chunk i computes on `stream`; smaller
 * batches run as one chunk on `stream`. The call is
 * stream-ordered: once `stream` has passed it, out_host holds the result.
 * Each chunk is routed on its own, so the router's split of H (and with it
 * the summation order of the FP32 logits) follows the chunk size.
 * Workspace: BEAM_MOE_OP_FORWARD_HOST bytes (the forward workspace of one
 * chunk plus two device staging buffers each for x and out). Calls that
 * share a workspace must not overlap.
 */
#define BEAM_MOE_HOST_CHUNK 8192
BEAM_MOE_API beam_moe_status beam_moe_forward_host(const beam_moe_cfg* cfg, int64_t T,
                                                   const uint16_t* x_host, const float* w_router,
                                                   const float* bias, const uint16_t* w13,
                                                   const uint16_t* w2, uint16_t* out_host,
                                                   void* ws, size_t ws_bytes, void* stream);

/* The same with NVFP4 experts (beam_moe_forward_nvfp4 per chunk).
 * Workspace: BEAM_MOE_OP_FORWARD_NVFP4_HOST bytes. */
BEAM_MOE_API beam_moe_status beam_moe_forward_nvfp4_host(
    const beam_moe_cfg* cfg, int64_t T, const uint16_t* x_host, const float* w_router,
    const float* bias, const beam_moe_nvfp4_experts* experts, uint16_t* out_host, void* ws,
    size_t ws_bytes, void* stream);

/*
 * Quantise `rows` rows of K fp32 values (device, K a multiple of 16) to
 * NVFP4 with tensor scale g, as beam_moe_forward_nvfp4 quantises x and h:
 * codes [rows][K/2] and scales row-major [rows][K/16] (device outputs).
 */
BEAM_MOE_API beam_moe_status beam_moe_nvfp4_quantize(int64_t rows, int64_t K, const float* v,
                                                     float g, uint8_t* codes, uint8_t* scales,
                                                     void* stream);

/*
 * Inspection of intermediates. beam_moe_forward_stages runs the stages of
 * beam_moe_forward up to and including `last_stage` (0 router GEMM, 1 top-k
 * and chunk counts, 2 scan, 3 permute, 4 gate/up grouped GEMM, 5 down grouped
 * GEMM, 6 combine; the numbering of the stage trace below) and leaves every
 * intermediate in the workspace; with last_stage = 6 it is beam_moe_forward
 * without the optional route outputs. out may be NULL unless last_stage is 6.
 * beam_moe_workspace_layout reports where the intermediates sit for T tokens
 * on the current device (byte offsets from the start of ws):
 *   counts  [E] int32          rows routed to each expert
 *   offsets [E+1] int32        first permuted row of each expert
 *   ids, w  [T][K] int32/fp32  routes and combine weights (S included)
 *   pos     [T][K] int32       permuted row of each (token, slot): the rows of
 *                              an expert are contiguous from offsets[e], in
 *                              ascending token order
 *   xp      [T*K][H] bf16      permuted token rows (valid after stage 3 and
 *                              until stage 5 overwrites them with y)
 *   h       [T*K][I] bf16      silu(g) * u of each permuted row (after stage 4)
 *   y       [T*K][H] fp32      down projection of each permuted row (after
 *                              stage 5; the same bytes as xp)
 * op must be BEAM_MOE_OP_ROUTE (only the routing arrays are meaningful) or
 * BEAM_MOE_OP_FORWARD. These calls exist for tests and debugging.
 */
typedef struct beam_moe_ws_layout {
  int64_t counts, offsets, ids, w, pos, xp, h, y; /* byte offsets in ws         */
  int32_t router_splits; /* slices of H whose FP32 partial logits are added  */
  int32_t router_tc;     /* 1: the router GEMM runs on tensor cores           */
  int32_t pair_gateup;   /* 1: gate/up grouped GEMM on CTA pairs              */
  int32_t pair_down;     /* 1: down grouped GEMM on CTA pairs                 */
  int32_t light_rows;    /* with CTA pairs: experts with at most this many
                            rows run on one-CTA tiles, after the CTA-pair
                            GEMMs (they only stream weights); 0: none       */
} beam_moe_ws_layout;
BEAM_MOE_API beam_moe_status beam_moe_workspace_layout(const beam_moe_cfg* cfg, int64_t T,
                                                       beam_moe_op op,
                                                       beam_moe_ws_layout* layout);
BEAM_MOE_API beam_moe_status beam_moe_forward_stages(
    const beam_moe_cfg* cfg, int64_t T, const uint16_t* x, const float* w_router,
    const float* bias, const uint16_t* w13, const uint16_t* w2, uint16_t* out,
    int32_t last_stage, void* ws, size_t ws_bytes, void* stream);

/*
 * Stage timing. A trace records CUDA events around each stage of the calls
 * it is passed to: slot i of stage s is the time of that stage in the i-th
 * traced call since the last reset. Stages: 0 router GEMM, 1 top-k and
 * chunk counts, 2 scan, 3 permute, 4 gate/up grouped GEMM, 5 down grouped
 * GEMM, 6 combine (a GEMM stage holds both of its launches when light
 * experts run on one-CTA tiles). beam_moe_trace_read synchronizes the
 * recorded events.
 */
#define BEAM_MOE_N_STAGES 7
typedef struct beam_moe_trace beam_moe_trace;
BEAM_MOE_API beam_moe_status beam_moe_trace_create(int32_t capacity, beam_moe_trace** out);
BEAM_MOE_API beam_moe_status beam_moe_trace_destroy(beam_moe_trace* trace);
BEAM_MOE_API beam_moe_status beam_moe_trace_reset(beam_moe_trace* trace);
/* ms[i * BEAM_MOE_N_STAGES + s] for i < *n_calls (at most capacity). */
BEAM_MOE_API beam_moe_status beam_moe_trace_read(beam_moe_trace* trace, float* ms, int32_t* n_calls);
BEAM_MOE_API beam_moe_status beam_moe_forward_nvfp4_traced(
    const beam_moe_cfg* cfg, int64_t T, const uint16_t* x, const float* w_router,
    const float* bias, const beam_moe_nvfp4_experts* experts, uint16_t* out, int32_t* topk_ids,
    float* topk_w, int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream,
    beam_moe_trace* trace);
BEAM_MOE_API beam_moe_status beam_moe_forward_traced(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                        const float* w_router, const float* bias,
                                        const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                                        int32_t* topk_ids, float* topk_w,
                                        int32_t* expert_counts, void* ws, size_t ws_bytes,
                                        void* stream, beam_moe_trace* trace);

/*
 * Expert parallelism. `world` ranks (one per GPU) each hold E / world
 * consecutive experts and route their own tokens; the block's arithmetic is
 * beam_moe_forward's, split over the ranks (the DEP / all-to-all layout the
 * vLLM recipe and DeepEP use for Beam, "Welcome Beam" and the vLLM recipe).
 * A rank calls, in order:
 *   1 beam_moe_ep_route     routes its T tokens, writes counts [E] (device)
 *   -                       the caller all-gathers counts into counts_all
 *                           [world][E] on the host
 *   2 beam_moe_ep_plan      (host) where this rank's rows land in every
 *                           owner's receive buffer, and what it receives
 *   3 beam_moe_ep_dispatch  writes its token rows and their return
 *                           addresses into the owners' workspaces and
 *                           counts each row on its owner's arrival counter
 *                           of the row's expert (system-scope atomics)
 *   4 beam_moe_ep_experts   grouped GEMMs over the received rows, each y row
 *                           written back into its source rank's workspace
 *                           (from the down GEMM's epilogue when it runs on
 *                           CTA pairs, else by a copy kernel after it). No
 *                           barrier is needed before it: the gate/up GEMM
 *                           starts on an expert's rows once its arrival
 *                           counter reaches recv_counts, so it overlaps the
 *                           other ranks' dispatch
 *   -                       barrier: every rank's experts call has completed
 *   5 beam_moe_ep_combine   out[t] = sum_k w[t][k] y[t][k], fixed k order
 * The arrival wait is the one place a kernel waits for another rank. It is
 * bounded: after 1 s without the rows it sets status bit 0x1000 and goes on
 * with whatever the buffer holds. Ranks must therefore run on different GPUs
 * (or, when several share one GPU, be ordered by the caller so that every
 * dispatch has completed before any experts call starts: kernels of
 * different processes on one GPU need not run at the same time). The route
 * call clears the rank's arrival counters; no rank may dispatch to it before
 * the counts of that route call have been gathered.
 * peer_ws[r] is rank r's workspace as a pointer this rank's GPU can store
 * to (NVLink peer memory; the same allocation when r == rank). Every rank's
 * workspace has the same size and layout (same cfg, world, t_max,
 * recv_cap); routes, returned rows and scratch stay in it from route to
 * combine. Rank r owns experts [r E / world, (r + 1) E / world).
 */
typedef struct beam_moe_ep_cfg {
  int32_t world;    /* ranks, 1..8, dividing n_experts                        */
  int32_t rank;     /* this rank, 0..world-1                                  */
  int64_t t_max;    /* most tokens a rank routes in one call                  */
  int64_t recv_cap; /* rows a rank's receive buffer holds (beam_moe_ep_plan
                       fails when any rank would receive more)                 */
} beam_moe_ep_cfg;
BEAM_MOE_API beam_moe_status beam_moe_ep_workspace_size(const beam_moe_cfg* cfg,
                                                        const beam_moe_ep_cfg* ep,
                                                        size_t* bytes);
/* counts [E] int32, device (out): this rank's tokens routed to each expert. */
BEAM_MOE_API beam_moe_status beam_moe_ep_route(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                               int64_t T, const uint16_t* x,
                                               const float* w_router, const float* bias,
                                               int32_t* counts, void* ws, size_t ws_bytes,
                                               void* stream);
/* Host only. counts_all [world][E] int32 (host): every rank's counts.
 * send_base [E] int32 (host, out): first row, in the owner's receive buffer,
 * of this rank's rows for each expert (its rows for an expert are in token
 * order; sources follow one another in rank order). recv_counts [E/world]
 * int32 (host, out): rows this rank receives per local expert; *recv_rows
 * their sum. Fails with BEAM_MOE_ERR_WORKSPACE_TOO_SMALL if any rank would
 * receive more than recv_cap rows (every rank reaches the same result). */
BEAM_MOE_API beam_moe_status beam_moe_ep_plan(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                              const int32_t* counts_all, int32_t* send_base,
                                              int32_t* recv_counts, int64_t* recv_rows);
/* x [T][H] bf16, device: the tokens routed by beam_moe_ep_route (same T).
 * send_base [E] int32, device: beam_moe_ep_plan's, copied to the device.
 * peer_ws [world] (host array of device pointers). */
BEAM_MOE_API beam_moe_status beam_moe_ep_dispatch(const beam_moe_cfg* cfg,
                                                  const beam_moe_ep_cfg* ep, int64_t T,
                                                  const uint16_t* x, const int32_t* send_base,
                                                  void* const* peer_ws, void* ws,
                                                  size_t ws_bytes, void* stream);
/* recv_counts [E/world] int32 (host): beam_moe_ep_plan's. w13, w2: this
 * rank's experts only ([E/world][2I][H], [E/world][H][I] bf16, device). */
BEAM_MOE_API beam_moe_status beam_moe_ep_experts(const beam_moe_cfg* cfg,
                                                 const beam_moe_ep_cfg* ep,
                                                 const int32_t* recv_counts,
                                                 const uint16_t* w13, const uint16_t* w2,
                                                 void* const* peer_ws, void* ws,
                                                 size_t ws_bytes, void* stream);
/* out [T][H] bf16, device (same T as the route call). */
BEAM_MOE_API beam_moe_status beam_moe_ep_combine(const beam_moe_cfg* cfg,
                                                 const beam_moe_ep_cfg* ep, int64_t T,
                                                 uint16_t* out, void* ws, size_t ws_bytes,
                                                 void* stream);

/*
 * Peer workspaces across processes (one process per GPU), through CUDA IPC.
 * Each rank exports its workspace once, the ranks exchange the handles (any
 * all-gather of these bytes; sizeof(beam_moe_ep_handle) is fixed), and each
 * rank imports every other rank's handle to get the peer_ws pointers the
 * dispatch and experts calls store through.
 *   beam_moe_ep_export  ws: this rank's workspace, device memory from
 *                       cudaMalloc (torch's default allocator qualifies; the
 *                       virtual-memory allocator's expandable segments do
 *                       not), at least ws_bytes long. Fills *handle: the IPC
 *                       handle of the allocation holding ws, ws's offset in
 *                       it, ws_bytes, the device ordinal and the process id.
 *   beam_moe_ep_import  opens another process's handle on the current device
 *                       (peer access is enabled as needed) and returns its
 *                       workspace in *peer_ws. A handle this process exported
 *                       is refused (BEAM_MOE_ERR_INVALID_ARG): use the local
 *                       pointer for your own rank. ws_bytes must not exceed
 *                       the exported size.
 *   beam_moe_ep_release closes what beam_moe_ep_import opened (peer_ws as it
 *                       returned it, with the same handle). Release every
 *                       peer before the exporting process frees or exits.
 * These calls synchronize with the device as CUDA IPC does; make them once at
 * set-up, not per step.
 */
typedef struct beam_moe_ep_handle {
  uint8_t ipc[64];  /* cudaIpcMemHandle_t of the allocation holding ws        */
  int64_t offset;   /* ws minus the allocation's base, bytes                  */
  int64_t bytes;    /* exported workspace size                                */
  int32_t device;   /* exporting device ordinal                               */
  int32_t pid;      /* exporting process                                      */
} beam_moe_ep_handle;
BEAM_MOE_API beam_moe_status beam_moe_ep_export(void* ws, size_t ws_bytes,
                                                beam_moe_ep_handle* handle);
BEAM_MOE_API beam_moe_status beam_moe_ep_import(const beam_moe_ep_handle* handle,
                                                size_t ws_bytes, void** peer_ws);
BEAM_MOE_API beam_moe_status beam_moe_ep_release(const beam_moe_ep_handle* handle,
                                                 void* peer_ws);

/*
 * Synchronizes `stream`, then reads and clears the device status word in the
 * workspace. *device_flags (may be NULL) receives the raw bits: 0x1 producer,
 * 0x2 MMA issuer, 0x4 epilogue gave up a bounded wait; 0x100 an expert id
 * outside [0, E) reached the dispatch; 0x200 beam_moe_selftest_wait's wait ran
 * out; 0x400 a received row's return address named no rank or slot (the row
 * is not stored; only inconsistent recv_counts lead there); 0x800 a
 * dispatched row's place in its owner's receive buffer fell outside
 * [0, recv_cap) (the row is not stored; send_base from another step's plan
 * leads there); 0x1000 an expert's received rows did not all arrive within
 * 1 s of the experts call's gate/up GEMM asking for them (recv_counts larger
 * than what the ranks dispatched, or a rank that never dispatched). Returns
 * BEAM_MOE_ERR_DEVICE_TIMEOUT
 * if any bit was set, BEAM_MOE_ERR_CUDA if the stream reports an error.
 */
BEAM_MOE_API beam_moe_status beam_moe_check(void* ws, size_t ws_bytes, void* stream, uint32_t* device_flags);

/*
 * Device self-check of the failure path: one thread waits on an mbarrier that
 * nothing completes; after limit_ms (1..1000) the wait gives up, sets status
 * bit 0x200 in the workspace's status word and the kernel returns, exactly as
 * a tensor-core kernel of this library does when one of its bounded waits
 * runs out. beam_moe_check then reports BEAM_MOE_ERR_DEVICE_TIMEOUT with that
 * bit, and the context stays usable. ws: at least 256 bytes, device.
 */
BEAM_MOE_API beam_moe_status beam_moe_selftest_wait(void* ws, size_t ws_bytes, int32_t limit_ms,
                                                    void* stream);

/* Static description of a status code. */
BEAM_MOE_API const char* beam_moe_status_string(beam_moe_status status);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H */
