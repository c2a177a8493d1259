// api.cu - host side of the C ABI declared in include/beam_moe.h: argument
// validation, the workspace layout, TMA descriptor encoding and the launch
// sequence of one Beam MoE block forward. Nothing here allocates device
// memory; nothing here synchronizes except beam_moe_check / trace reads.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <initializer_list>
#include <mutex>
#include <new>
#include <vector>

#include "internal.h"

extern "C" BEAM_MOE_API beam_moe_status beam_moe_workspace_size(const beam_moe_cfg*, int64_t, beam_moe_op,
                                                   size_t*);

namespace beam {

int device_sm_count() {
  static PerDevice cached;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const cudaError_t err = cached.get(dev, &sms, [dev](int* v) {
    if (cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || *v <= 0)
      *v = 148;
    return cudaSuccess;
  });
  return err == cudaSuccess ? sms : 148;
}

int router_split_k(int64_t T, int H, int E, int sms);

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Token tile of the grouped GEMMs: the smallest supported N that covers about
// 1.25x the mean rows per expert (T K / E), so most experts need one tile.
static int pick_bn(int64_t T, int K, int E) {
  const double mean = (double)T * K / E;
  const int opts[5] = {16, 32, 64, 128, 256};
  for (int b : opts)
    if (b >= 1.25 * mean) return b;
  return 256;
}

Layout make_layout(const beam_moe_cfg& c, int64_t T, int sms, bool allow_tc) {
  Layout L;
  memset(&L, 0, sizeof(L));
  const int E = c.n_experts, K = c.top_k, H = c.hidden, I = c.inter;
  L.T = T;
  L.A = T * K;
  L.nchunks = (int)((T + kChunk - 1) / kChunk);
  L.router_tc = (allow_tc && c.router_tc == 1 && router_tc_supported(c)) ? 1 : 0;
  if (L.router_tc) {
    const int nkb = H / 64;
    L.router_kper = router_tc_kper(T, H, E, sms);
    L.split_k = (nkb + L.router_kper - 1) / L.router_kper;
  } else {
    L.split_k = router_split_k(T, H, E, sms);
  }
  L.bn = pick_bn(T, K, E);
  // CTA pairs halve the token-row bytes each SM reads per weight byte and
  // double-buffer the accumulator. They run with 256-token tiles, which the
  // tile choice above reaches once experts average more than about 102 rows
  // (measured: prefill at 128 rows is faster on pairs for both GEMMs); below
  // that the GEMMs stream weights and one CTA per tile is enough.
  const double mean_rows = (double)T * K / E;
  const bool pair_ok = L.bn == 256 && pair_gemm_supported(c);
  L.pair_gateup = (pair_ok && mean_rows >= 64.0) ? 1 : 0;
  L.pair_down = (pair_ok && mean_rows >= 64.0) ? 1 : 0;
  // Experts with few rows only stream their weights; a pair tile of 256
  // weight rows does that at about 0.7 of HBM, the one-CTA kernel (128
  // weight rows, one 64-token tile) close to 1. With pairs on, such experts
  // run there, after the others.
  L.light_max = L.pair_gateup ? kLightRows : 0;
  L.light_bn = kLightRows;

  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) {
    o = align_up(o, align);
    size_t at = o;
    o += bytes;
    return at;
  };
  L.status = take(256, 256);
  L.counts = take(sizeof(int32_t) * E, 256);
  L.offsets = take(sizeof(int32_t) * (E + 1), 256);
  L.nb_off = take(sizeof(int32_t) * (E + 1), 256);
  L.nb2_off = take(sizeof(int32_t) * (E + 1), 256);
  L.nbl_off = take(sizeof(int32_t) * (E + 1), 256);
  L.ids = take(sizeof(int32_t) * (size_t)L.A, 256);
  L.w = take(sizeof(float) * (size_t)L.A, 256);
  L.pos = take(sizeof(int32_t) * (size_t)L.A, 256);
  L.chunk_cnt = take(sizeof(int32_t) * (size_t)L.nchunks * E, 256);
  L.chunk_mask = take(sizeof(uint32_t) * (size_t)L.nchunks * E * kChunkWords, 256);
  L.logits = take(sizeof(float) * (size_t)L.split_k * T * E, 256);
  L.w3 = L.router_tc ? take(2 * 3 * (size_t)E * H, 1024) : 0;
  L.route_end = align_up(o, 256);
  // permuted rows (bf16) during gate/up, then the down output y (fp32)
  L.xp = take(4 * (size_t)L.A * H, 1024);
  L.h = take(2 * (size_t)L.A * I, 1024);
  L.total = align_up(o, 256);
  return L;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor [rows][cols], box {box_cols, box_rows}, 128-byte swizzle,
// zero fill outside the tensor.
cudaError_t encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                                uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D byte tensor [rows][cols], box {box_cols, box_rows}, 128-byte swizzle.
cudaError_t encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                              uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// W13 [E][2I][H] seen as 5-D {H, 16, 2, I/16, E} (k, row in a 16-row block,
// gate/up, block, expert): a box {64, 16, 2, 4, 1} lands in shared memory as
// 128 rows ordered gate 0-15, up 0-15, gate 16-31, up 16-31, ... of 64
// consecutive intermediate indices.
cudaError_t encode_tmap_w13_interleaved(CUtensorMap* map, const void* w13, uint64_t H, uint64_t I,
                                        uint64_t E) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[5] = {H, 16, 2, I / 16, E};
  const cuuint64_t strides[4] = {H * 2, I * H * 2, 16 * H * 2, 2 * I * H * 2};
  const cuuint32_t box[5] = {64, 16, 2, 4, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(w13), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace beam

using beam::Layout;

// ------------------------------------------------------------- validation
static beam_moe_status check_cfg(const beam_moe_cfg* c) {
  if (!c) return BEAM_MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->n_group <= 0 ||
      c->topk_group <= 0 || c->top_k <= 0)
    return BEAM_MOE_ERR_INVALID_ARG;
  if (c->renormalize != 0 && c->renormalize != 1) return BEAM_MOE_ERR_INVALID_ARG;
  if (c->bias_mode != 0 && c->bias_mode != 1) return BEAM_MOE_ERR_INVALID_ARG;
  if (c->router_tc != 0 && c->router_tc != 1) return BEAM_MOE_ERR_INVALID_ARG;
  if (!isfinite(c->routed_scale)) return BEAM_MOE_ERR_INVALID_ARG;
  if (c->n_experts % c->n_group != 0 || c->topk_group > c->n_group) return BEAM_MOE_ERR_INVALID_ARG;
  const int gs = c->n_experts / c->n_group;
  if (c->top_k > c->topk_group * gs) return BEAM_MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 != 0 || c->inter % 128 != 0) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->hidden > 65536 || c->inter > 65536) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  if (c->n_experts > 512 || c->top_k > 32 || gs < 2) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  // the top-k warp gives each lane `per` consecutive experts of one group
  const int E = c->n_experts;
  const int per = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : E <= 256 ? 8 : 16;
  if (gs % per != 0) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  const int lg = gs / per;
  if (lg > 32 || (lg & (lg - 1)) != 0) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  return BEAM_MOE_OK;
}

static beam_moe_status check_T(const beam_moe_cfg* c, int64_t T) {
  if (T < 0) return BEAM_MOE_ERR_INVALID_ARG;
  // permuted rows are addressed with 32-bit ints and TMA row coordinates
  if (T * (int64_t)c->top_k > (int64_t)1 << 30) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  return BEAM_MOE_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define BEAM_TRY(expr)                          \
  do {                                          \
    beam_moe_status s_ = (expr);                \
    if (s_ != BEAM_MOE_OK) return s_;           \
  } while (0)

#define BEAM_CUDA(expr)                         \
  do {                                          \
    if ((expr) != cudaSuccess) return BEAM_MOE_ERR_CUDA; \
  } while (0)

// ------------------------------------------------------------------ trace
struct beam_moe_trace {
  int capacity;
  int n;
  std::vector<cudaEvent_t> ev;  // capacity * (stages + 1)
};

namespace {

struct Recorder {
  beam_moe_trace* tr;
  cudaStream_t st;
  int slot;
  bool on;
  Recorder(beam_moe_trace* t, cudaStream_t s) : tr(t), st(s), slot(-1), on(false) {
    if (tr && tr->n < tr->capacity) {
      slot = tr->n;
      on = true;
    }
  }
  cudaError_t mark(int i) {
    if (!on) return cudaSuccess;
    return cudaEventRecord(tr->ev[(size_t)slot * (BEAM_MOE_N_STAGES + 1) + i], st);
  }
  void done() {
    if (on) tr->n++;
  }
};

// Host-only checks, run before any CUDA call: configuration, T, workspace
// pointer, alignment and size. The size bound is the device-independent one
// beam_moe_workspace_size reports.
beam_moe_status common_checks(const beam_moe_cfg* cfg, int64_t T, void* ws, size_t ws_bytes,
                              beam_moe_op op) {
  BEAM_TRY(check_cfg(cfg));
  BEAM_TRY(check_T(cfg, T));
  if (T == 0) return BEAM_MOE_OK;
  if (!ws) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return BEAM_MOE_ERR_ALIGNMENT;
  size_t need = 0;
  BEAM_TRY(beam_moe_workspace_size(cfg, T, op, &need));
  if (ws_bytes < need) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  return BEAM_MOE_OK;
}

beam_moe_status check_ptrs(std::initializer_list<const void*> required,
                           std::initializer_list<const void*> optional) {
  for (const void* p : required)
    if (!p) return BEAM_MOE_ERR_INVALID_ARG;
  for (const void* p : required)
    if (!aligned16(p)) return BEAM_MOE_ERR_ALIGNMENT;
  for (const void* p : optional)
    if (p && !aligned16(p)) return BEAM_MOE_ERR_ALIGNMENT;
  return BEAM_MOE_OK;
}

// Layout for the current device (the first CUDA call of every entry point).
beam_moe_status plan(const beam_moe_cfg* cfg, int64_t T, Layout* L) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  *L = beam::make_layout(*cfg, T, beam::device_sm_count());
  return BEAM_MOE_OK;
}

// Stages 2..last of a forward (scan, permute, gate/up, down, combine).
beam_moe_status expert_path(const beam_moe_cfg* cfg, const Layout& L, const uint16_t* x,
                            const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                            int32_t* counts_out, char* ws, cudaStream_t st, Recorder& rec,
                            int last = 6) {
  BEAM_CUDA(beam::launch_scan(*cfg, L, ws, counts_out, st));
  BEAM_CUDA(rec.mark(3));
  if (last < 3) return BEAM_MOE_OK;
  BEAM_CUDA(beam::launch_permute(*cfg, L, x, ws, st));
  BEAM_CUDA(rec.mark(4));
  if (last < 4) return BEAM_MOE_OK;
  BEAM_CUDA(L.pair_gateup ? beam::launch_gateup_pair(*cfg, L, w13, ws, st)
                          : beam::launch_gateup(*cfg, L, w13, ws, st));
  if (L.light_max) BEAM_CUDA(beam::launch_gateup_light(*cfg, L, w13, ws, st));
  BEAM_CUDA(rec.mark(5));
  if (last < 5) return BEAM_MOE_OK;
  BEAM_CUDA(L.pair_down ? beam::launch_down_pair(*cfg, L, w2, ws, st)
                        : beam::launch_down(*cfg, L, w2, ws, st));
  if (L.light_max) BEAM_CUDA(beam::launch_down_light(*cfg, L, w2, ws, st));
  BEAM_CUDA(rec.mark(6));
  if (last < 6) return BEAM_MOE_OK;
  BEAM_CUDA(beam::launch_combine(*cfg, L, out, ws, st));
  BEAM_CUDA(rec.mark(7));
  return BEAM_MOE_OK;
}

// A forward through stage `last` (6: the whole block).
beam_moe_status forward_impl(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                             const float* w_router, const float* bias, const uint16_t* w13,
                             const uint16_t* w2, uint16_t* out, int32_t* topk_ids, float* topk_w,
                             int32_t* expert_counts, void* ws, size_t ws_bytes, void* stream,
                             beam_moe_trace* trace, int last = 6) {
  BEAM_TRY(common_checks(cfg, T, ws, ws_bytes, BEAM_MOE_OP_FORWARD));
  if (last < 0 || last > 6) return BEAM_MOE_ERR_INVALID_ARG;
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({x, w_router, w13, w2}, {bias, topk_ids, topk_w, expert_counts, out}));
  if (last == 6 && !out) return BEAM_MOE_ERR_INVALID_ARG;
  Layout L;
  BEAM_TRY(plan(cfg, T, &L));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  Recorder rec(last == 6 ? trace : nullptr, st);
  BEAM_CUDA(cudaMemsetAsync(w + L.status, 0, 256, st));
  BEAM_CUDA(rec.mark(0));
  BEAM_CUDA(beam::launch_router_logits(*cfg, L, x, w_router, w, st));
  BEAM_CUDA(rec.mark(1));
  if (last >= 1) {
    BEAM_CUDA(beam::launch_router_topk(*cfg, L, bias, w, st));
    BEAM_CUDA(rec.mark(2));
  }
  if (last >= 2) BEAM_TRY(expert_path(cfg, L, x, w13, w2, out, expert_counts, w, st, rec, last));
  if (last >= 1) BEAM_CUDA(beam::launch_copy_routes(*cfg, L, topk_ids, topk_w, w, st));
  rec.done();
  return BEAM_MOE_OK;
}

bool positive_finite(float v) { return isfinite(v) && v > 0.0f; }

beam_moe_status forward_nvfp4_impl(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                   const float* w_router, const float* bias,
                                   const beam_moe_nvfp4_experts* ex, uint16_t* out,
                                   int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                                   void* ws, size_t ws_bytes, void* stream,
                                   beam_moe_trace* trace) {
  BEAM_TRY(common_checks(cfg, T, ws, ws_bytes, BEAM_MOE_OP_FORWARD_NVFP4));
  if (T == 0) return BEAM_MOE_OK;
  if (!ex) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(check_ptrs({x, w_router, ex->w13_codes, ex->w13_scales, ex->w2_codes, ex->w2_scales,
                       out},
                      {bias, topk_ids, topk_w, expert_counts}));
  if (!positive_finite(ex->w13_scale) || !positive_finite(ex->w2_scale) ||
      !positive_finite(ex->x_scale) || !positive_finite(ex->h_scale))
    return BEAM_MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  const beam::Fp4Layout F = beam::make_layout_nvfp4(*cfg, T, beam::device_sm_count());
  const Layout& L = F.base;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  Recorder rec(trace, st);
  BEAM_CUDA(cudaMemsetAsync(w + L.status, 0, 256, st));
  BEAM_CUDA(rec.mark(0));
  BEAM_CUDA(beam::launch_router_logits(*cfg, L, x, w_router, w, st));
  BEAM_CUDA(rec.mark(1));
  BEAM_CUDA(beam::launch_router_topk(*cfg, L, bias, w, st));
  BEAM_CUDA(rec.mark(2));
  BEAM_CUDA(beam::launch_scan(*cfg, L, w, expert_counts, st));
  BEAM_CUDA(rec.mark(3));
  BEAM_CUDA(beam::launch_permute_nvfp4(*cfg, F, x, ex->x_scale, w, st));
  BEAM_CUDA(rec.mark(4));
  BEAM_CUDA(beam::launch_gateup_nvfp4(*cfg, F, *ex, w, st));
  BEAM_CUDA(rec.mark(5));
  BEAM_CUDA(F.pair_down ? beam::launch_down_nvfp4_pair(*cfg, F, *ex, w, st)
                        : beam::launch_down_nvfp4(*cfg, F, *ex, w, st));
  BEAM_CUDA(rec.mark(6));
  BEAM_CUDA(beam::launch_combine(*cfg, L, out, w, st));
  BEAM_CUDA(rec.mark(7));
  BEAM_CUDA(beam::launch_copy_routes(*cfg, L, topk_ids, topk_w, w, st));
  rec.done();
  return BEAM_MOE_OK;
}

// ------------------------------------------------------------ host buffers
// Chunking of a forward on host buffers: chunks of BEAM_MOE_HOST_CHUNK tokens
// once there are at least two, else one chunk; bf16 batches of at least
// 8 x BEAM_MOE_HOST_CHUNK tokens take chunks twice as large, because every
// chunk streams all touched experts once (20 GB in bf16) and at 8192 tokens
// that costs about 13 % of the compute. The chunk's forward workspace is
// sized for the larger of the full and the last chunk (the router's split of
// H, and with it the partial-logit buffer, is not monotone in T).
struct HostPlan {
  int64_t chunk, n_chunks;
  size_t fwd_bytes;  // forward workspace of one chunk
  size_t buf_bytes;  // one staging buffer: chunk x H bf16
  int n_bufs;        // staging buffers per direction
  size_t total;
};

beam_moe_status host_plan(const beam_moe_cfg* cfg, int64_t T, beam_moe_op fwd_op, HostPlan* hp) {
  const int64_t c = BEAM_MOE_HOST_CHUNK;
  hp->chunk = T < 2 * c ? T : ((fwd_op == BEAM_MOE_OP_FORWARD && T >= 8 * c) ? 2 * c : c);
  hp->n_chunks = (T + hp->chunk - 1) / hp->chunk;
  const int64_t last = T - (hp->n_chunks - 1) * hp->chunk;
  size_t a = 0, b = 0;
  BEAM_TRY(beam_moe_workspace_size(cfg, hp->chunk, fwd_op, &a));
  BEAM_TRY(beam_moe_workspace_size(cfg, last, fwd_op, &b));
  hp->fwd_bytes = beam::align_up(a > b ? a : b, 1024);
  hp->buf_bytes = beam::align_up((size_t)hp->chunk * cfg->hidden * 2, 1024);
  hp->n_bufs = hp->n_chunks > 1 ? 2 : 1;
  hp->total = hp->fwd_bytes + 2 * (size_t)hp->n_bufs * hp->buf_bytes;
  return BEAM_MOE_OK;
}

// Runs forward(Tc, x_dev, out_dev, fwd_ws, fwd_bytes, stream) per chunk. With
// several chunks, a chunk's upload waits until the forward two chunks back
// has read its staging buffer, its forward waits for its upload and for the
// download two chunks back, and its download waits for its forward. The
// caller's stream finally waits for the last download.
template <class Fwd>
beam_moe_status host_pipeline(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x_host,
                              uint16_t* out_host, char* ws, const HostPlan& hp,
                              cudaStream_t st, Fwd forward) {
  const int64_t H = cfg->hidden;
  uint16_t* xb[2];
  uint16_t* ob[2];
  for (int b = 0; b < hp.n_bufs; ++b) {
    xb[b] = reinterpret_cast<uint16_t*>(ws + hp.fwd_bytes + b * hp.buf_bytes);
    ob[b] = reinterpret_cast<uint16_t*>(ws + hp.fwd_bytes + (hp.n_bufs + b) * hp.buf_bytes);
  }
  if (hp.n_chunks == 1) {
    BEAM_CUDA(cudaMemcpyAsync(xb[0], x_host, (size_t)T * H * 2, cudaMemcpyHostToDevice, st));
    BEAM_TRY(forward(T, xb[0], ob[0], ws, hp.fwd_bytes, st));
    BEAM_CUDA(cudaMemcpyAsync(out_host, ob[0], (size_t)T * H * 2, cudaMemcpyDeviceToHost, st));
    return BEAM_MOE_OK;
  }
  // streams and events of this call; their destruction is deferred by the
  // runtime until the work that uses them has completed
  struct Res {
    cudaStream_t up = nullptr, down = nullptr;
    cudaEvent_t ev[8] = {};
    ~Res() {
      for (cudaEvent_t e : ev)
        if (e) cudaEventDestroy(e);
      if (up) cudaStreamDestroy(up);
      if (down) cudaStreamDestroy(down);
    }
  } r;
  BEAM_CUDA(cudaStreamCreateWithFlags(&r.up, cudaStreamNonBlocking));
  BEAM_CUDA(cudaStreamCreateWithFlags(&r.down, cudaStreamNonBlocking));
  for (cudaEvent_t& e : r.ev) BEAM_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  cudaEvent_t start = r.ev[0], done = r.ev[1];
  cudaEvent_t* uploaded = r.ev + 2;    // [2] staged x of a chunk is on the device
  cudaEvent_t* computed = r.ev + 4;    // [2] a chunk's forward has finished
  cudaEvent_t* downloaded = r.ev + 6;  // [2] a chunk's out has reached the host
  BEAM_CUDA(cudaEventRecord(start, st));  // the copies start after earlier work on st
  BEAM_CUDA(cudaStreamWaitEvent(r.up, start, 0));
  BEAM_CUDA(cudaStreamWaitEvent(r.down, start, 0));
  for (int64_t i = 0; i < hp.n_chunks; ++i) {
    const int b = (int)(i & 1);
    const int64_t t0 = i * hp.chunk;
    const int64_t tc = (T - t0) < hp.chunk ? (T - t0) : hp.chunk;
    const size_t bytes = (size_t)tc * H * 2;
    if (i >= 2) BEAM_CUDA(cudaStreamWaitEvent(r.up, computed[b], 0));
    BEAM_CUDA(cudaMemcpyAsync(xb[b], x_host + t0 * H, bytes, cudaMemcpyHostToDevice, r.up));
    BEAM_CUDA(cudaEventRecord(uploaded[b], r.up));
    BEAM_CUDA(cudaStreamWaitEvent(st, uploaded[b], 0));
    if (i >= 2) BEAM_CUDA(cudaStreamWaitEvent(st, downloaded[b], 0));
    BEAM_TRY(forward(tc, xb[b], ob[b], ws, hp.fwd_bytes, st));
    BEAM_CUDA(cudaEventRecord(computed[b], st));
    BEAM_CUDA(cudaStreamWaitEvent(r.down, computed[b], 0));
    BEAM_CUDA(cudaMemcpyAsync(out_host + t0 * H, ob[b], bytes, cudaMemcpyDeviceToHost, r.down));
    BEAM_CUDA(cudaEventRecord(downloaded[b], r.down));
  }
  BEAM_CUDA(cudaEventRecord(done, r.down));
  BEAM_CUDA(cudaStreamWaitEvent(st, done, 0));
  return BEAM_MOE_OK;
}

beam_moe_status host_checks(const beam_moe_cfg* cfg, int64_t T, const void* x_host,
                            const void* out_host, void* ws, size_t ws_bytes, beam_moe_op op,
                            HostPlan* hp) {
  BEAM_TRY(check_cfg(cfg));
  BEAM_TRY(check_T(cfg, T));
  if (T == 0) return BEAM_MOE_OK;
  if (!x_host || !out_host || !ws) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return BEAM_MOE_ERR_ALIGNMENT;
  BEAM_TRY(host_plan(cfg, T,
                     op == BEAM_MOE_OP_FORWARD_HOST ? BEAM_MOE_OP_FORWARD
                                                    : BEAM_MOE_OP_FORWARD_NVFP4,
                     hp));
  if (ws_bytes < hp->total) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  return BEAM_MOE_OK;
}

}  // namespace

extern "C" {

beam_moe_status beam_moe_forward_host(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x_host,
                                      const float* w_router, const float* bias,
                                      const uint16_t* w13, const uint16_t* w2, uint16_t* out_host,
                                      void* ws, size_t ws_bytes, void* stream) {
  HostPlan hp;
  BEAM_TRY(host_checks(cfg, T, x_host, out_host, ws, ws_bytes, BEAM_MOE_OP_FORWARD_HOST, &hp));
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({w_router, w13, w2}, {bias}));
  return host_pipeline(
      cfg, T, x_host, out_host, static_cast<char*>(ws), hp,
      reinterpret_cast<cudaStream_t>(stream),
      [&](int64_t tc, const uint16_t* xd, uint16_t* od, char* fws, size_t fb, cudaStream_t s) {
        return forward_impl(cfg, tc, xd, w_router, bias, w13, w2, od, nullptr, nullptr, nullptr,
                            fws, fb, s, nullptr);
      });
}

beam_moe_status beam_moe_forward_nvfp4_host(const beam_moe_cfg* cfg, int64_t T,
                                            const uint16_t* x_host, const float* w_router,
                                            const float* bias,
                                            const beam_moe_nvfp4_experts* experts,
                                            uint16_t* out_host, void* ws, size_t ws_bytes,
                                            void* stream) {
  if (cfg && !beam::nvfp4_supported(*cfg)) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  HostPlan hp;
  BEAM_TRY(
      host_checks(cfg, T, x_host, out_host, ws, ws_bytes, BEAM_MOE_OP_FORWARD_NVFP4_HOST, &hp));
  if (T == 0) return BEAM_MOE_OK;
  if (!experts) return BEAM_MOE_ERR_INVALID_ARG;
  return host_pipeline(
      cfg, T, x_host, out_host, static_cast<char*>(ws), hp,
      reinterpret_cast<cudaStream_t>(stream),
      [&](int64_t tc, const uint16_t* xd, uint16_t* od, char* fws, size_t fb, cudaStream_t s) {
        return forward_nvfp4_impl(cfg, tc, xd, w_router, bias, experts, od, nullptr, nullptr,
                                  nullptr, fws, fb, s, nullptr);
      });
}

beam_moe_status beam_moe_forward_nvfp4(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                       const float* w_router, const float* bias,
                                       const beam_moe_nvfp4_experts* experts, uint16_t* out,
                                       int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                                       void* ws, size_t ws_bytes, void* stream) {
  return forward_nvfp4_impl(cfg, T, x, w_router, bias, experts, out, topk_ids, topk_w,
                            expert_counts, ws, ws_bytes, stream, nullptr);
}

beam_moe_status beam_moe_forward_nvfp4_traced(const beam_moe_cfg* cfg, int64_t T,
                                              const uint16_t* x, const float* w_router,
                                              const float* bias,
                                              const beam_moe_nvfp4_experts* experts,
                                              uint16_t* out, int32_t* topk_ids, float* topk_w,
                                              int32_t* expert_counts, void* ws, size_t ws_bytes,
                                              void* stream, beam_moe_trace* trace) {
  if (!trace) return BEAM_MOE_ERR_INVALID_ARG;
  return forward_nvfp4_impl(cfg, T, x, w_router, bias, experts, out, topk_ids, topk_w,
                            expert_counts, ws, ws_bytes, stream, trace);
}

beam_moe_status beam_moe_nvfp4_quantize(int64_t rows, int64_t K, const float* v, float g,
                                        uint8_t* codes, uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || K % 16 != 0 || !positive_finite(g)) return BEAM_MOE_ERR_INVALID_ARG;
  if (rows == 0) return BEAM_MOE_OK;
  if (!v || !codes || !scales) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(codes) || !aligned16(scales)) return BEAM_MOE_ERR_ALIGNMENT;
  BEAM_CUDA(beam::launch_quantize_rows(rows, K, v, g, codes, scales,
                                       reinterpret_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_workspace_size(const beam_moe_cfg* cfg, int64_t T, beam_moe_op op,
                                        size_t* bytes) {
  BEAM_TRY(check_cfg(cfg));
  BEAM_TRY(check_T(cfg, T));
  if (!bytes || (op != BEAM_MOE_OP_ROUTE && op != BEAM_MOE_OP_FORWARD &&
                 op != BEAM_MOE_OP_FORWARD_NVFP4 && op != BEAM_MOE_OP_FORWARD_HOST &&
                 op != BEAM_MOE_OP_FORWARD_NVFP4_HOST))
    return BEAM_MOE_ERR_INVALID_ARG;
  if ((op == BEAM_MOE_OP_FORWARD_NVFP4 || op == BEAM_MOE_OP_FORWARD_NVFP4_HOST) &&
      !beam::nvfp4_supported(*cfg))
    return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) {
    *bytes = 0;
    return BEAM_MOE_OK;
  }
  if (op == BEAM_MOE_OP_FORWARD_HOST || op == BEAM_MOE_OP_FORWARD_NVFP4_HOST) {
    HostPlan hp;
    BEAM_TRY(host_plan(cfg, T,
                       op == BEAM_MOE_OP_FORWARD_HOST ? BEAM_MOE_OP_FORWARD
                                                      : BEAM_MOE_OP_FORWARD_NVFP4,
                       &hp));
    *bytes = hp.total;
    return BEAM_MOE_OK;
  }
  // Sized for the largest split-K any device could pick (148 SMs bound it for
  // B200; the 1024-SM bound keeps the size valid on any part).
  if (op == BEAM_MOE_OP_FORWARD_NVFP4) {
    *bytes = beam::make_layout_nvfp4(*cfg, T, 1024).base.total;
    return BEAM_MOE_OK;
  }
  Layout L = beam::make_layout(*cfg, T, 1024);
  *bytes = op == BEAM_MOE_OP_ROUTE ? L.route_end : L.total;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_route(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                               const float* w_router, const float* bias, int32_t* topk_ids,
                               float* topk_w, int32_t* expert_counts, void* ws, size_t ws_bytes,
                               void* stream) {
  BEAM_TRY(common_checks(cfg, T, ws, ws_bytes, BEAM_MOE_OP_ROUTE));
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({x, w_router, topk_ids, topk_w}, {bias, expert_counts}));
  Layout L;
  BEAM_TRY(plan(cfg, T, &L));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  BEAM_CUDA(cudaMemsetAsync(w + L.status, 0, 256, st));
  BEAM_CUDA(beam::launch_router_logits(*cfg, L, x, w_router, w, st));
  BEAM_CUDA(beam::launch_router_topk(*cfg, L, bias, w, st));
  if (expert_counts) BEAM_CUDA(beam::launch_scan(*cfg, L, w, expert_counts, st));
  BEAM_CUDA(beam::launch_copy_routes(*cfg, L, topk_ids, topk_w, w, st));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                 const float* w_router, const float* bias, const uint16_t* w13,
                                 const uint16_t* w2, uint16_t* out, int32_t* topk_ids,
                                 float* topk_w, int32_t* expert_counts, void* ws,
                                 size_t ws_bytes, void* stream) {
  return forward_impl(cfg, T, x, w_router, bias, w13, w2, out, topk_ids, topk_w, expert_counts,
                      ws, ws_bytes, stream, nullptr);
}

beam_moe_status beam_moe_forward_stages(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                        const float* w_router, const float* bias,
                                        const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                                        int32_t last_stage, void* ws, size_t ws_bytes,
                                        void* stream) {
  return forward_impl(cfg, T, x, w_router, bias, w13, w2, out, nullptr, nullptr, nullptr, ws,
                      ws_bytes, stream, nullptr, last_stage);
}

beam_moe_status beam_moe_workspace_layout(const beam_moe_cfg* cfg, int64_t T, beam_moe_op op,
                                          beam_moe_ws_layout* out) {
  BEAM_TRY(check_cfg(cfg));
  BEAM_TRY(check_T(cfg, T));
  if (!out || (op != BEAM_MOE_OP_ROUTE && op != BEAM_MOE_OP_FORWARD))
    return BEAM_MOE_ERR_INVALID_ARG;
  Layout L;
  BEAM_TRY(plan(cfg, T, &L));
  out->counts = (int64_t)L.counts;
  out->offsets = (int64_t)L.offsets;
  out->ids = (int64_t)L.ids;
  out->w = (int64_t)L.w;
  out->pos = (int64_t)L.pos;
  out->xp = (int64_t)L.xp;
  out->h = (int64_t)L.h;
  out->y = (int64_t)L.xp;
  out->router_splits = L.split_k;
  out->router_tc = L.router_tc;
  out->pair_gateup = L.pair_gateup;
  out->pair_down = L.pair_down;
  out->light_rows = L.light_max;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_forward_traced(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                        const float* w_router, const float* bias,
                                        const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                                        int32_t* topk_ids, float* topk_w,
                                        int32_t* expert_counts, void* ws, size_t ws_bytes,
                                        void* stream, beam_moe_trace* trace) {
  if (!trace) return BEAM_MOE_ERR_INVALID_ARG;
  return forward_impl(cfg, T, x, w_router, bias, w13, w2, out, topk_ids, topk_w, expert_counts,
                      ws, ws_bytes, stream, trace);
}

beam_moe_status beam_moe_forward_routed(const beam_moe_cfg* cfg, int64_t T, const uint16_t* x,
                                        const int32_t* topk_ids, const float* topk_w,
                                        const uint16_t* w13, const uint16_t* w2, uint16_t* out,
                                        int32_t* expert_counts, void* ws, size_t ws_bytes,
                                        void* stream) {
  BEAM_TRY(common_checks(cfg, T, ws, ws_bytes, BEAM_MOE_OP_FORWARD));
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({x, topk_ids, topk_w, w13, w2, out}, {expert_counts}));
  Layout L;
  BEAM_TRY(plan(cfg, T, &L));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  BEAM_CUDA(cudaMemsetAsync(w + L.status, 0, 256, st));
  BEAM_CUDA(beam::launch_routes_given(*cfg, L, topk_ids, topk_w, w, st));
  Recorder none(nullptr, st);
  return expert_path(cfg, L, x, w13, w2, out, expert_counts, w, st, none);
}

beam_moe_status beam_moe_trace_create(int32_t capacity, beam_moe_trace** out) {
  if (!out || capacity <= 0 || capacity > (1 << 20)) return BEAM_MOE_ERR_INVALID_ARG;
  beam_moe_trace* t = new (std::nothrow) beam_moe_trace;
  if (!t) return BEAM_MOE_ERR_INVALID_ARG;
  t->capacity = capacity;
  t->n = 0;
  t->ev.assign((size_t)capacity * (BEAM_MOE_N_STAGES + 1), nullptr);
  for (auto& e : t->ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      e = nullptr;
      beam_moe_trace_destroy(t);
      return BEAM_MOE_ERR_CUDA;
    }
  }
  *out = t;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_trace_destroy(beam_moe_trace* t) {
  if (!t) return BEAM_MOE_ERR_INVALID_ARG;
  for (auto& e : t->ev)
    if (e) cudaEventDestroy(e);
  delete t;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_trace_reset(beam_moe_trace* t) {
  if (!t) return BEAM_MOE_ERR_INVALID_ARG;
  t->n = 0;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_trace_read(beam_moe_trace* t, float* ms, int32_t* n_calls) {
  if (!t || !n_calls) return BEAM_MOE_ERR_INVALID_ARG;
  *n_calls = t->n;
  if (!ms) return BEAM_MOE_OK;
  for (int i = 0; i < t->n; ++i) {
    cudaEvent_t* ev = &t->ev[(size_t)i * (BEAM_MOE_N_STAGES + 1)];
    if (cudaEventSynchronize(ev[BEAM_MOE_N_STAGES]) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
    for (int s = 0; s < BEAM_MOE_N_STAGES; ++s)
      if (cudaEventElapsedTime(&ms[(size_t)i * BEAM_MOE_N_STAGES + s], ev[s], ev[s + 1]) !=
          cudaSuccess)
        return BEAM_MOE_ERR_CUDA;
  }
  return BEAM_MOE_OK;
}

// ------------------------------------------------------ expert parallelism
}  // extern "C"

namespace {

beam_moe_status ep_checks(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep) {
  BEAM_TRY(check_cfg(cfg));
  if (!ep) return BEAM_MOE_ERR_INVALID_ARG;
  if (ep->world < 1 || ep->world > 8 || ep->rank < 0 || ep->rank >= ep->world ||
      ep->t_max < 0 || ep->recv_cap < 0)
    return BEAM_MOE_ERR_INVALID_ARG;
  if (cfg->n_experts % ep->world != 0) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  // return addresses hold the source rank above 27 bits of token slot
  if (ep->t_max * cfg->top_k >= ((int64_t)1 << 27) || ep->recv_cap >= ((int64_t)1 << 31))
    return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  BEAM_TRY(check_T(cfg, ep->t_max));
  return BEAM_MOE_OK;
}

// The routing layout of T tokens, moved to start at `base` of the workspace;
// its status word is the workspace's first (shared with the expert stage).
Layout ep_routing(const beam_moe_cfg& c, int64_t T, int sms, size_t base) {
  Layout L = beam::make_layout(c, T, sms);
  size_t* f[] = {&L.counts, &L.offsets, &L.nb_off, &L.nb2_off, &L.nbl_off, &L.ids, &L.w, &L.pos,
                 &L.chunk_cnt, &L.chunk_mask, &L.logits, &L.w3, &L.route_end, &L.xp, &L.h,
                 &L.total};
  for (size_t* v : f) *v += base;
  L.status = 0;
  return L;
}

// Routing scratch for any T <= t_max. Its size is not monotone in T (the
// router's split over H depends on T), so take the maximum: every T up to
// 4096, then the last T of every 128-token block (both routers' token tiles
// are whole 128-token blocks there, so within one block the split is fixed
// and the size grows with T).
size_t ep_route_bytes_scan(const beam_moe_cfg& c, int64_t t_max) {
  size_t best = 0;
  for (int64_t t = 1; t <= t_max; t = (t < 4096 ? t + 1 : (t + 128) / 128 * 128)) {
    const Layout L = beam::make_layout(c, t, 1024);
    if (L.route_end > best) best = L.route_end;
    if (t >= 4096 && t + 128 > t_max && t != t_max) {
      const Layout M = beam::make_layout(c, t_max, 1024);
      if (M.route_end > best) best = M.route_end;
      break;
    }
  }
  return best;
}

// ep_route_bytes_scan's result, remembered per (configuration, t_max): every
// phase of an expert-parallel step checks its workspace size, and the scan
// walks thousands of layouts.
size_t ep_route_bytes(const beam_moe_cfg& c, int64_t t_max) {
  struct Entry {
    beam_moe_cfg cfg;
    int64_t t_max;
    size_t bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> seen;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : seen)
      if (e.t_max == t_max && memcmp(&e.cfg, &c, sizeof(c)) == 0) return e.bytes;
  }
  const size_t bytes = ep_route_bytes_scan(c, t_max);
  std::lock_guard<std::mutex> lock(mu);
  if (seen.size() < 64) seen.push_back({c, t_max, bytes});
  return bytes;
}

beam_moe_status ep_ws_checks(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep, void* ws,
                             size_t ws_bytes) {
  if (!ws) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return BEAM_MOE_ERR_ALIGNMENT;
  size_t need = 0;
  BEAM_TRY(beam_moe_ep_workspace_size(cfg, ep, &need));
  if (ws_bytes < need) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  return BEAM_MOE_OK;
}

}  // namespace

extern "C" {

beam_moe_status beam_moe_ep_workspace_size(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                           size_t* bytes) {
  BEAM_TRY(ep_checks(cfg, ep));
  if (!bytes) return BEAM_MOE_ERR_INVALID_ARG;
  const beam::EpLayout P = beam::make_ep_layout(*cfg, *ep);
  *bytes = P.route + ep_route_bytes(*cfg, ep->t_max);
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_route(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep, int64_t T,
                                  const uint16_t* x, const float* w_router, const float* bias,
                                  int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
  BEAM_TRY(ep_checks(cfg, ep));
  if (T < 0 || T > ep->t_max) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(ep_ws_checks(cfg, ep, ws, ws_bytes));
  BEAM_TRY(check_ptrs({counts}, {}));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  const beam::EpLayout P = beam::make_ep_layout(*cfg, *ep);
  BEAM_CUDA(cudaMemsetAsync(w, 0, 256, st));
  // arrival counters of this step: no rank dispatches here before the counts
  // of this call have been gathered
  BEAM_CUDA(cudaMemsetAsync(w + P.arrive, 0, 4 * (size_t)(cfg->n_experts / ep->world), st));
  if (T == 0) {
    BEAM_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * cfg->n_experts, st));
    return BEAM_MOE_OK;
  }
  BEAM_TRY(check_ptrs({x, w_router}, {bias}));
  const Layout L = ep_routing(*cfg, T, beam::device_sm_count(), P.route);
  BEAM_CUDA(beam::launch_router_logits(*cfg, L, x, w_router, w, st));
  BEAM_CUDA(beam::launch_router_topk(*cfg, L, bias, w, st));
  BEAM_CUDA(beam::launch_scan(*cfg, L, w, counts, st));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_plan(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                 const int32_t* counts_all, int32_t* send_base,
                                 int32_t* recv_counts, int64_t* recv_rows) {
  BEAM_TRY(ep_checks(cfg, ep));
  if (!counts_all || !send_base || !recv_counts || !recv_rows) return BEAM_MOE_ERR_INVALID_ARG;
  const int E = cfg->n_experts, W = ep->world, El = E / W;
  for (int s = 0; s < W; ++s) {
    int64_t sum = 0;
    for (int e = 0; e < E; ++e) {
      const int32_t v = counts_all[(size_t)s * E + e];
      if (v < 0) return BEAM_MOE_ERR_INVALID_ARG;
      sum += v;
    }
    if (sum > ep->t_max * cfg->top_k) return BEAM_MOE_ERR_INVALID_ARG;
  }
  // owner o's receive buffer: local experts in order, each expert's rows
  // from source 0, then source 1, ...
  for (int o = 0; o < W; ++o) {
    int64_t row = 0;
    for (int j = 0; j < El; ++j) {
      const int e = o * El + j;
      int64_t got = 0;
      for (int s = 0; s < W; ++s) {
        if (s == ep->rank) send_base[e] = (int32_t)(row + got);
        got += counts_all[(size_t)s * E + e];
      }
      if (o == ep->rank) recv_counts[j] = (int32_t)got;
      row += got;
    }
    if (row > ep->recv_cap) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (o == ep->rank) *recv_rows = row;
  }
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_dispatch(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                     int64_t T, const uint16_t* x, const int32_t* send_base,
                                     void* const* peer_ws, void* ws, size_t ws_bytes,
                                     void* stream) {
  BEAM_TRY(ep_checks(cfg, ep));
  if (T < 0 || T > ep->t_max) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(ep_ws_checks(cfg, ep, ws, ws_bytes));
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({x, send_base}, {}));
  if (!peer_ws) return BEAM_MOE_ERR_INVALID_ARG;
  for (int r = 0; r < ep->world; ++r)
    if (!peer_ws[r] || !aligned16(peer_ws[r])) return BEAM_MOE_ERR_INVALID_ARG;
  if (peer_ws[ep->rank] != ws) return BEAM_MOE_ERR_INVALID_ARG;
  const beam::EpLayout P = beam::make_ep_layout(*cfg, *ep);
  const Layout L = ep_routing(*cfg, T, beam::device_sm_count(), P.route);
  BEAM_CUDA(beam::launch_ep_dispatch(*cfg, *ep, P, L, x, send_base, peer_ws,
                                     static_cast<char*>(ws), reinterpret_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_experts(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                    const int32_t* recv_counts, const uint16_t* w13,
                                    const uint16_t* w2, void* const* peer_ws, void* ws,
                                    size_t ws_bytes, void* stream) {
  BEAM_TRY(ep_checks(cfg, ep));
  BEAM_TRY(ep_ws_checks(cfg, ep, ws, ws_bytes));
  if (!recv_counts || !peer_ws) return BEAM_MOE_ERR_INVALID_ARG;
  const int El = cfg->n_experts / ep->world;
  std::vector<int32_t> counts(El), offsets(El + 1), nb_off(El + 1);
  int64_t rows = 0;
  for (int j = 0; j < El; ++j) {
    if (recv_counts[j] < 0) return BEAM_MOE_ERR_INVALID_ARG;
    counts[j] = recv_counts[j];
    offsets[j] = (int32_t)rows;
    rows += recv_counts[j];
  }
  offsets[El] = (int32_t)rows;
  if (rows > ep->recv_cap) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  if (rows == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({w13, w2}, {}));
  for (int r = 0; r < ep->world; ++r)
    if (!peer_ws[r] || !aligned16(peer_ws[r])) return BEAM_MOE_ERR_INVALID_ARG;
  if (peer_ws[ep->rank] != ws) return BEAM_MOE_ERR_INVALID_ARG;
  // the received rows as the grouped GEMMs' permuted rows, over the local
  // experts; token tile and CTA pairs chosen as for a forward
  beam_moe_cfg lc = *cfg;
  lc.n_experts = El;
  const beam::EpLayout P = beam::make_ep_layout(*cfg, *ep);
  Layout L;
  memset(&L, 0, sizeof(L));
  L.A = rows;
  L.T = rows;
  L.bn = beam::pick_bn(rows, 1, El);
  const double mean = (double)rows / El;
  const bool pair_ok = L.bn == 256 && beam::pair_gemm_supported(lc);
  L.pair_gateup = L.pair_down = (pair_ok && mean >= 64.0) ? 1 : 0;
  L.status = P.status;
  L.counts = P.counts;
  L.offsets = P.offsets;
  L.nb_off = P.nb_off;
  L.xp = P.recv;
  L.h = P.h;
  L.arrive = P.arrive;  // gate/up waits for each expert's rows from the other ranks
  int32_t acc = 0;
  for (int j = 0; j < El; ++j) {
    nb_off[j] = acc;
    acc += (counts[j] + L.bn - 1) / L.bn;
  }
  nb_off[El] = acc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* w = static_cast<char*>(ws);
  BEAM_CUDA(cudaMemcpyAsync(w + P.counts, counts.data(), 4 * El, cudaMemcpyHostToDevice, st));
  BEAM_CUDA(cudaMemcpyAsync(w + P.offsets, offsets.data(), 4 * (El + 1), cudaMemcpyHostToDevice, st));
  BEAM_CUDA(cudaMemcpyAsync(w + P.nb_off, nb_off.data(), 4 * (El + 1), cudaMemcpyHostToDevice, st));
  BEAM_CUDA(cudaStreamSynchronize(st));  // the host arrays are this call's
  BEAM_CUDA(L.pair_gateup ? beam::launch_gateup_pair(lc, L, w13, w, st)
                          : beam::launch_gateup(lc, L, w13, w, st));
  if (L.pair_down) {
    // the down GEMM's epilogue stores every y row into its source's workspace
    beam::EpReturn ret;
    memset(&ret, 0, sizeof(ret));
    ret.src = reinterpret_cast<const int32_t*>(w + P.src);
    for (int r = 0; r < ep->world; ++r) ret.peer[r] = static_cast<char*>(peer_ws[r]);
    ret.yret_off = P.yret;
    ret.world = ep->world;
    ret.slots = ep->t_max * cfg->top_k;
    BEAM_CUDA(beam::launch_down_pair(lc, L, w2, w, st, &ret));
  } else {
    BEAM_CUDA(beam::launch_down(lc, L, w2, w, st));
    BEAM_CUDA(beam::launch_ep_return(*cfg, *ep, P, rows, peer_ws, w, st));
  }
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_combine(const beam_moe_cfg* cfg, const beam_moe_ep_cfg* ep,
                                    int64_t T, uint16_t* out, void* ws, size_t ws_bytes,
                                    void* stream) {
  BEAM_TRY(ep_checks(cfg, ep));
  if (T < 0 || T > ep->t_max) return BEAM_MOE_ERR_INVALID_ARG;
  BEAM_TRY(ep_ws_checks(cfg, ep, ws, ws_bytes));
  if (T == 0) return BEAM_MOE_OK;
  BEAM_TRY(check_ptrs({out}, {}));
  const beam::EpLayout P = beam::make_ep_layout(*cfg, *ep);
  const Layout L = ep_routing(*cfg, T, beam::device_sm_count(), P.route);
  char* w = static_cast<char*>(ws);
  BEAM_CUDA(beam::launch_combine_from(*cfg, T, reinterpret_cast<const float*>(w + P.yret),
                                      reinterpret_cast<const int32_t*>(w + L.pos),
                                      reinterpret_cast<const float*>(w + L.w), out,
                                      reinterpret_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_check(void* ws, size_t ws_bytes, void* stream, uint32_t* device_flags) {
  if (!ws || ws_bytes < 256) return BEAM_MOE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  uint32_t flags = 0;
  // The status word is the first 4 bytes of every workspace layout.
  if (cudaMemcpy(&flags, ws, sizeof(flags), cudaMemcpyDeviceToHost) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  if (cudaMemset(ws, 0, sizeof(flags)) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  if (device_flags) *device_flags = flags;
  return flags ? BEAM_MOE_ERR_DEVICE_TIMEOUT : BEAM_MOE_OK;
}

beam_moe_status beam_moe_selftest_wait(void* ws, size_t ws_bytes, int32_t limit_ms,
                                       void* stream) {
  if (!ws || ws_bytes < 256 || limit_ms < 1 || limit_ms > 1000) return BEAM_MOE_ERR_INVALID_ARG;
  if (!aligned16(ws)) return BEAM_MOE_ERR_ALIGNMENT;
  BEAM_CUDA(beam::launch_selftest_wait(static_cast<unsigned*>(ws), limit_ms,
                                       reinterpret_cast<cudaStream_t>(stream)));
  return BEAM_MOE_OK;
}

const char* beam_moe_status_string(beam_moe_status s) {
  switch (s) {
    case BEAM_MOE_OK: return "ok";
    case BEAM_MOE_ERR_INVALID_ARG: return "invalid argument";
    case BEAM_MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BEAM_MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case BEAM_MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case BEAM_MOE_ERR_CUDA: return "CUDA error";
    case BEAM_MOE_ERR_DEVICE_TIMEOUT: return "device-side check failed (bounded wait or bad id)";
  }
  return "unknown status";
}

}  // extern "C"
