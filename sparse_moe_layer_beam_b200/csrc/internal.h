// internal.h - shared declarations of the Beam MoE block library (not public).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "beam_moe.h"

namespace beam {

// Tokens per dispatch chunk: the stable per-expert rank of a token is counted
// inside its chunk with one bit per token.
constexpr int kChunk = 128;
constexpr int kChunkWords = kChunk / 32;

// Rows of weights per tensor-core tile (the MMA M dimension) and the K step
// of one pipeline stage (64 bf16 = one 128-byte swizzle row).
constexpr int kTileM = 128;
constexpr int kTileK = 64;
constexpr int kLightRows = 64;  // see Layout::light_max
constexpr int kTileCounterWord = 32;  // status-area word: the CTA-pair GEMMs' tile counter

// Status bits written by kernels into the workspace status word.
constexpr uint32_t kFlagProducer = 0x1;
constexpr uint32_t kFlagMma = 0x2;
constexpr uint32_t kFlagEpilogue = 0x4;
constexpr uint32_t kFlagBadExpert = 0x100;
constexpr uint32_t kFlagSelftest = 0x200;  // beam_moe_selftest_wait's wait ran out
constexpr uint32_t kFlagBadReturn = 0x400; // a received row's return address out of range
constexpr uint32_t kFlagBadDispatch = 0x800; // a dispatched row would land outside recv_cap
constexpr uint32_t kFlagArrival = 0x1000;    // an expert's received rows did not all arrive

// A value set up once per device (a kernel's shared-memory attribute, the
// number of CTA pairs that can be resident), for host code that launches on
// several devices from several threads. get() runs setup(&v) under the lock
// the first time it is asked for `dev`; a failed set-up is retried next time.
class PerDevice {
 public:
  static constexpr int kMaxDevices = 64;
  template <class F>
  cudaError_t get(int dev, int* out, F&& setup) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu_);
    if (!done_[dev]) {
      int v = 0;
      const cudaError_t err = setup(&v);
      if (err != cudaSuccess) return err;
      val_[dev] = v;
      done_[dev] = true;
    }
    *out = val_[dev];
    return cudaSuccess;
  }

 private:
  std::mutex mu_;
  int val_[kMaxDevices] = {};
  bool done_[kMaxDevices] = {};
};

// The current device's PerDevice value (cudaGetDevice, then get()).
template <class F>
cudaError_t per_device(PerDevice& pd, int* out, F&& setup) {
  int dev = 0;
  const cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  return pd.get(dev, out, setup);
}

// Byte offsets of every scratch array inside the caller's workspace.
struct Layout {
  int64_t T, A;     // tokens, assignments (T * K)
  int nchunks;      // ceil(T / kChunk)
  int split_k;      // router split-K factor (slices of partial logits)
  int router_tc;    // 1: router GEMM on tensor cores (router_tc.cu), 0: CUDA cores
  int router_kper;  // tensor-core router: K blocks of 64 per split
  int bn;           // token tile of the grouped GEMMs
  int pair_gateup; // 1: gate/up grouped GEMM on CTA pairs
  int pair_down;   // 1: down grouped GEMM on CTA pairs
  int light_max;   // with CTA pairs: experts with at most this many rows go to the
                   // one-CTA kernel instead (0: none)
  int light_bn;    // that kernel's token tile
  size_t status;    // uint32[64]
  size_t counts;    // int32[E]
  size_t offsets;   // int32[E + 1] first row of each expert in the permuted rows
  size_t nb_off;    // int32[E + 1] prefix of ceil(count / bn) (light experts: 0)
  size_t nb2_off;   // int32[E + 1] prefix of ceil(count / (2 bn))
  size_t nbl_off;   // int32[E + 1] prefix of ceil(count / light_bn) over the light experts
  size_t ids;       // int32[T * K]
  size_t w;         // float[T * K]
  size_t pos;       // int32[T * K] permuted row of each assignment
  size_t chunk_cnt; // int32[nchunks * E] first row of each (chunk, expert)
  size_t chunk_mask;// uint32[nchunks * E * kChunkWords]
  size_t logits;    // float[split_k * T * E] partial router logits
  size_t w3;        // bf16[3][E][H] exact three-way split of the router weights
  size_t route_end; // bytes needed by the routing op
  size_t xp;        // bf16[A * H] permuted rows; reused for the down output y, fp32[A * H]
  size_t h;         // bf16[A * I] SwiGLU activations
  size_t arrive;    // int32[E] rows of each expert arrived from other ranks (0: none to wait for)
  size_t total;     // bytes needed by the forward op
};

// The router GEMM runs on tensor cores only when the configuration asks for
// it (c.router_tc) and allow_tc is set; allow_tc = false keeps it on CUDA
// cores whatever the configuration says (no weight planes needed).
Layout make_layout(const beam_moe_cfg& c, int64_t T, int sms, bool allow_tc = true);

// NVFP4 path: the routing layout (token tiles of 128 rows, expert segments
// padded to them) plus quantised activations and their scales.
struct Fp4Layout {
  Layout base;    // routing arrays; base.xp holds the fp32 down output y
  int64_t rows;   // bound on the padded rows
  size_t xq;      // uint8[rows * H/2] quantised x, expert segments 128-row aligned
  size_t xsf;     // uint8[rows * H/16] their scales (atom layout)
  size_t hq;      // uint8[rows * I/2] quantised h
  size_t hsf;     // uint8[rows * I/16]
  int pair_down;  // 1: down GEMM on CTA pairs (nvfp4_2sm.cu)
};
Fp4Layout make_layout_nvfp4(const beam_moe_cfg& c, int64_t T, int sms);
bool nvfp4_supported(const beam_moe_cfg& c);
bool nvfp4_pair_supported(const beam_moe_cfg& c);

// Expert parallelism: byte offsets inside every rank's workspace (identical
// across ranks, so that peers can store into it). `route` is where the
// routing layout of the rank's own tokens starts.
// Expert parallelism: a received row's return address is its source rank
// << kEpSlotBits | its token slot (t K + k) on that rank.
constexpr int kEpMaxWorld = 8;
constexpr int kEpSlotBits = 27;

// Where the down GEMM on CTA pairs stores y. src == nullptr: the workspace's
// y rows. Otherwise each row goes straight to its source rank's returned-y
// buffer, peer[rank] + yret_off + slot * H floats (a peer store).
struct EpReturn {
  const int32_t* src;        // [rows] return address of every received row
  char* peer[kEpMaxWorld];   // every rank's workspace
  size_t yret_off;           // the returned-y buffer inside a workspace
  int world;                 // ranks; a return address names one of them
  int64_t slots;             // returned-y rows per rank (T_max K)
};

struct EpLayout {
  size_t status, recv, src, yret, h, counts, offsets, nb_off, arrive, route;
};
EpLayout make_ep_layout(const beam_moe_cfg& c, const beam_moe_ep_cfg& g);

// ---- launchers (each enqueues on `st`, returns cudaGetLastError()) --------
// EP: token rows and return addresses to the owners; y rows back to sources.
// L is the routing layout with offsets relative to ws.
cudaError_t launch_ep_dispatch(const beam_moe_cfg& c, const beam_moe_ep_cfg& g,
                               const EpLayout& P, const Layout& L, const uint16_t* x,
                               const int32_t* send_base, void* const* peer_ws, char* ws,
                               cudaStream_t st);
cudaError_t launch_ep_return(const beam_moe_cfg& c, const beam_moe_ep_cfg& g, const EpLayout& P,
                             int64_t rows, void* const* peer_ws, char* ws, cudaStream_t st);
cudaError_t launch_selftest_wait(unsigned* status, int limit_ms, cudaStream_t st);
cudaError_t launch_combine_from(const beam_moe_cfg& c, int64_t T, const float* y,
                                const int32_t* pos, const float* w, uint16_t* out,
                                cudaStream_t st);
// Router GEMM into the partial logits: the tensor-core kernel when
// L.router_tc, else the CUDA-core kernel. Either clears the dispatch bits.
cudaError_t launch_router_logits(const beam_moe_cfg& c, const Layout& L, const uint16_t* x,
                                 const float* w_router, char* ws, cudaStream_t st);
cudaError_t launch_router_tc(const beam_moe_cfg& c, const Layout& L, const uint16_t* x,
                             const float* w_router, char* ws, cudaStream_t st);
bool router_tc_supported(const beam_moe_cfg& c);
int router_tc_kper(int64_t T, int H, int E, int sms);
cudaError_t launch_router_topk(const beam_moe_cfg& c, const Layout& L, const float* bias,
                               char* ws, cudaStream_t st);
cudaError_t launch_routes_given(const beam_moe_cfg& c, const Layout& L, const int32_t* ids,
                                const float* w, char* ws, cudaStream_t st);
cudaError_t launch_scan(const beam_moe_cfg& c, const Layout& L, char* ws, int32_t* counts_out,
                        cudaStream_t st);
cudaError_t launch_permute(const beam_moe_cfg& c, const Layout& L, const uint16_t* x, char* ws,
                           cudaStream_t st);
cudaError_t launch_gateup(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13, char* ws,
                          cudaStream_t st);
// The one-CTA kernels over the light experts only (L.light_max > 0), after the
// CTA-pair kernels have done the others.
cudaError_t launch_gateup_light(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13,
                                char* ws, cudaStream_t st);
cudaError_t launch_down_light(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2,
                              char* ws, cudaStream_t st);
cudaError_t launch_down(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2, char* ws,
                        cudaStream_t st);
bool pair_gemm_supported(const beam_moe_cfg& c);
cudaError_t launch_gateup_pair(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13,
                               char* ws, cudaStream_t st);
cudaError_t launch_down_pair(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2,
                             char* ws, cudaStream_t st, const EpReturn* ret = nullptr);
cudaError_t launch_combine(const beam_moe_cfg& c, const Layout& L, uint16_t* out, char* ws,
                           cudaStream_t st);
cudaError_t launch_copy_routes(const beam_moe_cfg& c, const Layout& L, int32_t* ids_out,
                               float* w_out, char* ws, cudaStream_t st);

// Tensor-map encoding through the driver entry point (no link to libcuda).
cudaError_t encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                                uint32_t box_cols, uint32_t box_rows);

cudaError_t encode_tmap_w13_interleaved(CUtensorMap* map, const void* w13, uint64_t H, uint64_t I,
                                        uint64_t E);

cudaError_t encode_tmap_2d_u8(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                              uint32_t box_cols, uint32_t box_rows);
cudaError_t launch_permute_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F, const uint16_t* x,
                                 float gx, char* ws, cudaStream_t st);
cudaError_t launch_gateup_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F,
                                const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st);
cudaError_t launch_down_nvfp4_pair(const beam_moe_cfg& c, const Fp4Layout& F,
                                   const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st);
cudaError_t launch_down_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F,
                              const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st);
cudaError_t launch_quantize_rows(int64_t rows, int64_t K, const float* v, float g, uint8_t* codes,
                                 uint8_t* sf, cudaStream_t st);

int device_sm_count();

// Slices of a token's row that the per-token kernels (permute, combine) spread
// over a second grid dimension when there are few tokens: enough CTAs for
// about two per SM, at most one 128-thread pass of `work` items per slice.
inline int h_slices(int64_t T, int work) {
  const int64_t want = T > 0 ? (2 * (int64_t)device_sm_count() + T - 1) / T : 1;
  const int64_t most = (work + 127) / 128;
  return (int)(want < 1 ? 1 : (want > most ? most : want));
}

}  // namespace beam
