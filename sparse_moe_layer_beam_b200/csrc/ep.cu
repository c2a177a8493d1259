// ep.cu - the Beam MoE block with expert parallelism: world ranks (one per
// GPU), each holding E / world consecutive experts. The pages run Beam this
// way (vLLM DEP / MegaMoE, DeepEP dispatch and combine); the block's
// arithmetic is the same as beam_moe_forward's, split over the ranks:
//
//   route     each rank routes its own tokens (the router is replicated);
//   plan      (host) from every rank's per-expert counts, where each rank's
//             rows land in each owner's receive buffer;
//   dispatch  each rank writes its token rows straight into the owners'
//             receive buffers with peer stores (NVLink), plus the row's return
//             address (source rank, token slot), and counts every row on its
//             owner's per-expert arrival counter;
//   experts   each rank runs the grouped GEMMs over the rows it received,
//             starting on an expert's rows as soon as its counter shows them
//             all (no barrier between dispatch and experts), and writes every
//             y row back into its source rank's buffer;
//   combine   each rank sums its tokens' K returned rows with the weights.
//
// The caller orders the other phases across ranks (an all-gather of the
// counts between route and plan, a barrier after experts). The gate/up GEMM's
// wait for arrivals is the only place a kernel waits for another rank; it is
// bounded (1 s, then status bit kFlagArrival). Every rank's workspace has the
// same layout, so a peer's buffer is its workspace pointer plus a fixed
// offset: [status][receive rows: cap x H x 4 bytes, bf16 on arrival, fp32 y
// after the down GEMM][return addresses: cap x int32][returned y: T_max K x H
// fp32][h: cap x I bf16][local expert counts, offsets, token-tile prefix]
// [arrival counters: E / world int32][routing scratch].
#include <string.h>

#include "internal.h"

namespace beam {
namespace {

constexpr int kMaxWorld = kEpMaxWorld;
constexpr int kSlotBits = kEpSlotBits;

struct Peers {
  char* ws[kMaxWorld];
};

size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

EpLayout make_ep_layout(const beam_moe_cfg& c, const beam_moe_ep_cfg& g) {
  EpLayout P;
  const size_t H = c.hidden, I = c.inter, K = c.top_k;
  const int El = c.n_experts / g.world;
  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) {
    o = up(o, align);
    size_t at = o;
    o += bytes;
    return at;
  };
  P.status = take(256, 256);
  P.recv = take((size_t)g.recv_cap * H * 4, 1024);
  P.src = take((size_t)g.recv_cap * 4, 256);
  P.yret = take((size_t)g.t_max * K * H * 4, 1024);
  P.h = take((size_t)g.recv_cap * I * 2, 1024);
  P.counts = take(4 * (size_t)El, 256);
  P.offsets = take(4 * (size_t)(El + 1), 256);
  P.nb_off = take(4 * (size_t)(El + 1), 256);
  P.arrive = take(4 * (size_t)El, 256);
  P.route = up(o, 1024);
  return P;
}

namespace {

// One CTA per local token: the K return addresses and combine positions,
// then the token's row copied to each owner's receive buffer and counted on
// the owner's arrival counter of its expert (after a system-scope fence, so
// an owner that sees the count sees the row). A row whose
// place in the owner's buffer falls outside [0, recv_cap) (send_base from
// another step's plan, for instance) is never stored: it is dropped, its
// combine position is -1 and status bit kFlagBadDispatch is set.
__global__ void __launch_bounds__(128) ep_dispatch_kernel(
    const uint16_t* __restrict__ x, int H, int K, int E, int El, int rank,
    const int32_t* __restrict__ ids, const int32_t* __restrict__ chunk_base,
    const uint32_t* __restrict__ chunk_mask, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ send_base, int32_t* __restrict__ pos,
    const __grid_constant__ Peers peers,
    size_t recv_off, size_t src_off, size_t arrive_off, int64_t recv_cap, unsigned* status) {
  __shared__ uint16_t* s_dst[32];
  __shared__ int32_t* s_arrive[32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < K) {
    const size_t slot = (size_t)t * K + tid;
    const int e = ids[slot];
    uint16_t* dst = nullptr;
    int32_t* arr = nullptr;
    if (e >= 0 && e < E) {
      const int c = t / kChunk, tl = t - c * kChunk;
      const uint32_t* m = chunk_mask + ((size_t)c * E + e) * kChunkWords;
      int r = 0;
      for (int wd = 0; wd < (tl >> 5); ++wd) r += __popc(m[wd]);
      r += __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
      const int64_t row =
          (int64_t)send_base[e] + (chunk_base[(size_t)c * E + e] + r - offsets[e]);
      if (row >= 0 && row < recv_cap) {
        char* peer = peers.ws[e / El];
        dst = reinterpret_cast<uint16_t*>(peer + recv_off) + (size_t)row * H;
        arr = reinterpret_cast<int32_t*>(peer + arrive_off) + (e % El);
        reinterpret_cast<int32_t*>(peer + src_off)[row] = (rank << kSlotBits) | (int)slot;
        pos[slot] = (int)slot;
      } else {
        atomicOr(status, kFlagBadDispatch);
        pos[slot] = -1;
      }
    } else {
      pos[slot] = -1;
    }
    s_dst[tid] = dst;
    s_arrive[tid] = arr;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  for (int k = 0; k < K; ++k) {
    uint4* d = reinterpret_cast<uint4*>(s_dst[k]);
    if (!d) continue;
    for (int v = tid; v < H / 8; v += 128) d[v] = __ldg(src + v);
  }
  // every store of this CTA reaches the owners (other GPUs) before its count
  __threadfence_system();
  __syncthreads();
  if (tid < K && s_arrive[tid]) atomicAdd_system(s_arrive[tid], 1);
}

// Every received y row back to its source rank's returned-y buffer.
__global__ void __launch_bounds__(128) ep_return_kernel(const float* __restrict__ y, int H,
                                                        int64_t rows,
                                                        const int32_t* __restrict__ src,
                                                        const __grid_constant__ Peers peers,
                                                        size_t yret_off, int world,
                                                        int64_t slots, unsigned* status) {
  for (int64_t i = blockIdx.x; i < rows; i += gridDim.x) {
    const uint32_t code = (uint32_t)src[i];
    const int s = (int)(code >> kSlotBits);
    const size_t slot = code & ((1u << kSlotBits) - 1u);
    if (s >= world || (int64_t)slot >= slots) {  // never stored through
      if (threadIdx.x == 0) atomicOr(status, kFlagBadReturn);
      continue;
    }
    float4* d = reinterpret_cast<float4*>(peers.ws[s] + yret_off) + slot * (H / 4);
    const float4* from = reinterpret_cast<const float4*>(y + (size_t)i * H);
    for (int v = threadIdx.x; v < H / 4; v += 128) d[v] = __ldg(from + v);
  }
  __threadfence_system();  // the sources combine these rows on other GPUs
}

}  // namespace

cudaError_t launch_ep_dispatch(const beam_moe_cfg& c, const beam_moe_ep_cfg& g,
                               const EpLayout& P, const Layout& L, const uint16_t* x,
                               const int32_t* send_base, void* const* peer_ws, char* ws,
                               cudaStream_t st) {
  if (L.T == 0) return cudaSuccess;
  char* wr = ws;  // L's offsets are relative to the workspace
  Peers peers;
  memset(&peers, 0, sizeof(peers));
  for (int r = 0; r < g.world; ++r) peers.ws[r] = static_cast<char*>(peer_ws[r]);
  ep_dispatch_kernel<<<(unsigned)L.T, 128, 0, st>>>(
      x, c.hidden, c.top_k, c.n_experts, c.n_experts / g.world, g.rank,
      reinterpret_cast<const int32_t*>(wr + L.ids), reinterpret_cast<const int32_t*>(wr + L.chunk_cnt),
      reinterpret_cast<const uint32_t*>(wr + L.chunk_mask),
      reinterpret_cast<const int32_t*>(wr + L.offsets), send_base,
      reinterpret_cast<int32_t*>(wr + L.pos), peers, P.recv, P.src, P.arrive, g.recv_cap,
      reinterpret_cast<unsigned*>(wr + P.status));
  return cudaGetLastError();
}

cudaError_t launch_ep_return(const beam_moe_cfg& c, const beam_moe_ep_cfg& g, const EpLayout& P,
                             int64_t rows, void* const* peer_ws, char* ws, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  Peers peers;
  memset(&peers, 0, sizeof(peers));
  for (int r = 0; r < g.world; ++r) peers.ws[r] = static_cast<char*>(peer_ws[r]);
  const int64_t grid = rows < 8L * device_sm_count() ? rows : 8L * device_sm_count();
  ep_return_kernel<<<(unsigned)grid, 128, 0, st>>>(
      reinterpret_cast<const float*>(ws + P.recv), c.hidden, rows,
      reinterpret_cast<const int32_t*>(ws + P.src), peers, P.yret, g.world,
      g.t_max * c.top_k, reinterpret_cast<unsigned*>(ws + P.status));
  return cudaGetLastError();
}

}  // namespace beam
