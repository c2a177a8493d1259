// ep_ipc.cu - peer workspaces across processes for expert parallelism:
// export a workspace as a CUDA IPC handle (plus its offset inside the
// allocation that holds it), open another process's handle, close it. The
// pages run Beam's experts over several GPUs (vLLM DEP, DeepEP all-to-all);
// how the ranks reach each other's buffers is this library's design.
#include <string.h>
#include <unistd.h>

#include <mutex>

#include "internal.h"

namespace {

typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the runtime's driver entry point (the library
// does not link libcuda).
AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  });
  return fn;
}

static_assert(sizeof(cudaIpcMemHandle_t) == 64, "CUDA IPC handles are 64 bytes");

}  // namespace

extern "C" {

beam_moe_status beam_moe_ep_export(void* ws, size_t ws_bytes, beam_moe_ep_handle* handle) {
  if (!ws || !handle || ws_bytes == 0) return BEAM_MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return BEAM_MOE_ERR_ALIGNMENT;
  AddressRangeFn range = address_range_fn();
  if (!range) return BEAM_MOE_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ws)) != CUDA_SUCCESS)
    return BEAM_MOE_ERR_INVALID_ARG;  // not device memory of this context
  const uintptr_t off = reinterpret_cast<uintptr_t>(ws) - static_cast<uintptr_t>(base);
  if (off + ws_bytes > size) return BEAM_MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_MOE_ERR_CUDA;
  memset(handle, 0, sizeof(*handle));
  memcpy(handle->ipc, &h, sizeof(h));
  handle->offset = (int64_t)off;
  handle->bytes = (int64_t)ws_bytes;
  handle->device = dev;
  handle->pid = (int32_t)getpid();
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_import(const beam_moe_ep_handle* handle, size_t ws_bytes,
                                   void** peer_ws) {
  if (!handle || !peer_ws || handle->offset < 0 || handle->bytes <= 0)
    return BEAM_MOE_ERR_INVALID_ARG;
  if ((int64_t)ws_bytes > handle->bytes) return BEAM_MOE_ERR_WORKSPACE_TOO_SMALL;
  if (handle->pid == (int32_t)getpid()) return BEAM_MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->ipc, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return BEAM_MOE_ERR_CUDA;
  *peer_ws = static_cast<char*>(base) + handle->offset;
  return BEAM_MOE_OK;
}

beam_moe_status beam_moe_ep_release(const beam_moe_ep_handle* handle, void* peer_ws) {
  if (!handle || !peer_ws || handle->offset < 0) return BEAM_MOE_ERR_INVALID_ARG;
  void* base = static_cast<char*>(peer_ws) - handle->offset;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? BEAM_MOE_OK : BEAM_MOE_ERR_CUDA;
}

}  // extern "C"
