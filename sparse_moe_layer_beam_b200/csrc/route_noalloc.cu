// route_noalloc.cu - routing entry point for callers that cannot allocate
// device memory (see beam_moe_route_noalloc in include/beam_moe.h).
//
// It runs the same router kernels as beam_moe_route, but its scratch is a
// fixed array in the library's own device memory instead of a caller
// workspace. Host code must not hand the array's name to a kernel: on the host
// that name is only a stand-in for the symbol. The device address is looked up
// with cudaGetSymbolAddress once per device, with that device current, on the
// first call made while it is current.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = BEAM_MOE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Shared by every call on a device; it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_scratch_mu;
char* g_scratch_ptr[kMaxDevices] = {};

beam_moe_status scratch_for_current_device(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BEAM_MOE_ERR_UNSUPPORTED_SHAPE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p)
      return BEAM_MOE_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<char*>(p);
  }
  *out = g_scratch_ptr[dev];
  return BEAM_MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" BEAM_MOE_API beam_moe_status beam_moe_route_noalloc(
    const beam_moe_cfg* cfg, int64_t T, const uint16_t* x, const float* w_router,
    const float* bias, int32_t* topk_ids, float* topk_w, int32_t* expert_counts, void* stream) {
  size_t unused = 0;
  beam_moe_status s = beam_moe_workspace_size(cfg, T, BEAM_MOE_OP_ROUTE, &unused);
  if (s != BEAM_MOE_OK) return s;  // configuration or T invalid
  if (T == 0) return BEAM_MOE_OK;
  if (T > BEAM_MOE_NOALLOC_MAX_TOKENS || cfg->n_experts > BEAM_MOE_NOALLOC_MAX_EXPERTS)
    return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  if (!x || !w_router || !topk_ids || !topk_w) return BEAM_MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, w_router, bias, topk_ids, topk_w, expert_counts};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return BEAM_MOE_ERR_ALIGNMENT;

  // Fewer router splits when the split partial sums would not fit.
  int sms = beam::device_sm_count();
  beam::Layout L = beam::make_layout(*cfg, T, sms, false);
  while (L.route_end > kScratchBytes && sms > 1) {
    sms /= 2;
    L = beam::make_layout(*cfg, T, sms, false);
  }
  if (L.route_end > kScratchBytes) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;

  char* ws = nullptr;
  s = scratch_for_current_device(&ws);
  if (s != BEAM_MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The only scratch that must start at zero is the status word; every other
  // array is written in full before it is read.
  if (cudaMemsetAsync(ws + L.status, 0, 256, st) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  if (beam::launch_router_logits(*cfg, L, x, w_router, ws, st) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  if (beam::launch_router_topk(*cfg, L, bias, ws, st) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  if (expert_counts && beam::launch_scan(*cfg, L, ws, expert_counts, st) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  if (beam::launch_copy_routes(*cfg, L, topk_ids, topk_w, ws, st) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  return BEAM_MOE_OK;
}
