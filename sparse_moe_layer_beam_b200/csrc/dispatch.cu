// dispatch.cu - token dispatch and combine of the Beam MoE block.
//
// The pages describe routing and combining ("Welcome Beam", section "Mixture
// of Experts": only 8 experts run per token; their outputs are combined with
// normalized weights and scaled by 2.5); grouping rows by expert so that every
// expert runs as one dense GEMM is this library's design.
//
//   scan     per-expert counts (popcounts of the chunk bits), first row of
//            each expert (exclusive scan),
//            the base row of every (chunk, expert) and the prefix of token
//            tiles per expert that the grouped GEMMs schedule from. All of it
//            stays on the device.
//   permute  row of assignment (t, k) = base(chunk of t, e) + number of
//            earlier tokens of the chunk routed to e (a popcount of the chunk
//            bits): rows of an expert are in ascending token order. Copies
//            x[t] to each of its K rows with 16-byte loads and stores.
//   combine  out[t] = sum_k w[t][k] * y[row(t, k)], k ascending, FP32 y and
//            FP32 accumulation, rounded once to bf16. No atomics.
#include <cuda_bf16.h>

#include "internal.h"

namespace beam {
namespace {

__device__ __forceinline__ int chunk_count(const uint32_t* __restrict__ bits, size_t i) {
  const uint4 m = __ldg(reinterpret_cast<const uint4*>(bits) + i);
  return __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
}

// Exclusive scan of v over threads 0..n-1 (n <= 1024); every thread of the
// block must call it. Returns the exclusive prefix, writes the total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += n;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += n;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of each warp
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_tot[warp] + inc - v;
  __syncthreads();
  return r;
}

// light_max > 0: experts with at most light_max rows get no bn-blocks in
// nb_off and ceil(count / lbn) blocks in nbl_off (the others none there).
__global__ void __launch_bounds__(1024) scan_kernel(const uint32_t* __restrict__ bits,
                                                    int32_t* __restrict__ chunk_base, int nchunks,
                                                    int E, int bn, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ nb_off,
                                                    int32_t* __restrict__ nb2_off,
                                                    int light_max, int lbn,
                                                    int32_t* __restrict__ nbl_off,
                                                    int32_t* __restrict__ counts_out) {
  __shared__ int32_t part[1024];   // per (team member, expert) partial counts
  __shared__ int32_t s_off[512];   // first row of each expert
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t total[4];
  const int tid = threadIdx.x;
  const int tpe = 1024 / E;  // threads per expert (E <= 512)
  const int e = tid % E, j = tid / E;
  const bool act = j < tpe;
  const int L = (nchunks + tpe - 1) / tpe;
  const int c0 = j * L, c1 = min(nchunks, c0 + L);
  int sum = 0;
  if (act)
    for (int c = c0; c < c1; ++c) sum += chunk_count(bits, (size_t)c * E + e);
  part[tid] = sum;
  __syncthreads();
  int tot = 0;
  if (tid < E)
    for (int q = 0; q < tpe; ++q) tot += part[q * E + tid];
  const bool light = tid < E && light_max > 0 && tot <= light_max;
  const int off = block_exclusive_scan(tid < E ? tot : 0, warp_tot, &total[0]);
  const int nbo =
      block_exclusive_scan(tid < E && !light ? (tot + bn - 1) / bn : 0, warp_tot, &total[1]);
  const int nb2o =
      block_exclusive_scan(tid < E ? (tot + 2 * bn - 1) / (2 * bn) : 0, warp_tot, &total[2]);
  const int nblo = block_exclusive_scan(light ? (tot + lbn - 1) / lbn : 0, warp_tot, &total[3]);
  if (tid < E) {
    s_off[tid] = off;
    offsets[tid] = off;
    nb_off[tid] = nbo;
    nb2_off[tid] = nb2o;
    nbl_off[tid] = nblo;
    counts[tid] = tot;
    if (counts_out) counts_out[tid] = tot;
  }
  if (tid == 0) {
    offsets[E] = total[0];
    nb_off[E] = total[1];
    nb2_off[E] = total[2];
    nbl_off[E] = total[3];
  }
  __syncthreads();
  if (act) {
    int run = s_off[e];
    for (int q = 0; q < j; ++q) run += part[q * E + e];
    for (int c = c0; c < c1; ++c) {
      const size_t i = (size_t)c * E + e;
      chunk_base[i] = run;
      run += chunk_count(bits, i);
    }
  }
}

__global__ void __launch_bounds__(128) permute_kernel(const uint16_t* __restrict__ x, int H, int K,
                                                      int E, const int32_t* __restrict__ ids,
                                                      const int32_t* __restrict__ chunk_base,
                                                      const uint32_t* __restrict__ chunk_mask,
                                                      int32_t* __restrict__ pos,
                                                      uint16_t* __restrict__ xp) {
  __shared__ int s_pos[32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < K) {
    const int e = ids[(size_t)t * K + tid];
    int p = -1;
    if (e >= 0 && e < E) {
      const int c = t / kChunk, tl = t - c * kChunk;
      const uint32_t* m = chunk_mask + ((size_t)c * E + e) * kChunkWords;
      int rank = 0;
      for (int wd = 0; wd < (tl >> 5); ++wd) rank += __popc(m[wd]);
      rank += __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
      p = chunk_base[(size_t)c * E + e] + rank;
    }
    s_pos[tid] = p;
    if (blockIdx.y == 0) pos[(size_t)t * K + tid] = p;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const int nv = H / 8;
  for (int v = blockIdx.y * 128 + tid; v < nv; v += gridDim.y * 128) {  // this CTA's slice of H
    const uint4 d = __ldg(src + v);
    for (int k = 0; k < K; ++k) {
      const int p = s_pos[k];
      if (p >= 0) reinterpret_cast<uint4*>(xp + (size_t)p * H)[v] = d;
    }
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo), b = __float2bfloat16_rn(hi);
  return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ y, int H, int K,
                                                      const int32_t* __restrict__ pos,
                                                      const float* __restrict__ w,
                                                      uint16_t* __restrict__ out) {
  __shared__ int s_pos[32];
  __shared__ float s_w[32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < K) {
    s_pos[tid] = pos[(size_t)t * K + tid];
    s_w[tid] = w[(size_t)t * K + tid];
  }
  __syncthreads();
  const int nv = H / 8;
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)t * H);
  for (int v = blockIdx.y * 128 + tid; v < nv; v += gridDim.y * 128) {  // this CTA's slice of H
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) {
      const int p = s_pos[k];
      if (p < 0) continue;
      const float4* src = reinterpret_cast<const float4*>(y + (size_t)p * H) + 2 * v;
      const float4 a = __ldg(src), b = __ldg(src + 1);
      const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      const float wk = s_w[k];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(wk, f[i], acc[i]);
    }
    dst[v] = make_uint4(pack2(acc[0], acc[1]), pack2(acc[2], acc[3]), pack2(acc[4], acc[5]),
                        pack2(acc[6], acc[7]));
  }
}

}  // namespace

cudaError_t launch_scan(const beam_moe_cfg& c, const Layout& L, char* ws, int32_t* counts_out,
                        cudaStream_t st) {
  scan_kernel<<<1, 1024, 0, st>>>(reinterpret_cast<const uint32_t*>(ws + L.chunk_mask),
                                  reinterpret_cast<int32_t*>(ws + L.chunk_cnt), L.nchunks,
                                  c.n_experts, L.bn, reinterpret_cast<int32_t*>(ws + L.counts),
                                  reinterpret_cast<int32_t*>(ws + L.offsets),
                                  reinterpret_cast<int32_t*>(ws + L.nb_off),
                                  reinterpret_cast<int32_t*>(ws + L.nb2_off), L.light_max,
                                  L.light_bn, reinterpret_cast<int32_t*>(ws + L.nbl_off),
                                  counts_out);
  return cudaGetLastError();
}

cudaError_t launch_permute(const beam_moe_cfg& c, const Layout& L, const uint16_t* x, char* ws,
                           cudaStream_t st) {
  permute_kernel<<<dim3((unsigned)L.T, (unsigned)h_slices(L.T, c.hidden / 8)), 128, 0, st>>>(
      x, c.hidden, c.top_k, c.n_experts, reinterpret_cast<const int32_t*>(ws + L.ids),
      reinterpret_cast<const int32_t*>(ws + L.chunk_cnt),
      reinterpret_cast<const uint32_t*>(ws + L.chunk_mask), reinterpret_cast<int32_t*>(ws + L.pos),
      reinterpret_cast<uint16_t*>(ws + L.xp));
  return cudaGetLastError();
}

cudaError_t launch_combine(const beam_moe_cfg& c, const Layout& L, uint16_t* out, char* ws,
                           cudaStream_t st) {
  combine_kernel<<<dim3((unsigned)L.T, (unsigned)h_slices(L.T, c.hidden / 8)), 128, 0, st>>>(
      reinterpret_cast<const float*>(ws + L.xp), c.hidden, c.top_k,
      reinterpret_cast<const int32_t*>(ws + L.pos), reinterpret_cast<const float*>(ws + L.w), out);
  return cudaGetLastError();
}

cudaError_t launch_combine_from(const beam_moe_cfg& c, int64_t T, const float* y,
                                const int32_t* pos, const float* w, uint16_t* out,
                                cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  combine_kernel<<<dim3((unsigned)T, (unsigned)h_slices(T, c.hidden / 8)), 128, 0, st>>>(
      y, c.hidden, c.top_k, pos, w, out);
  return cudaGetLastError();
}

cudaError_t launch_copy_routes(const beam_moe_cfg& c, const Layout& L, int32_t* ids_out,
                               float* w_out, char* ws, cudaStream_t st) {
  const size_t n = (size_t)L.A;
  if (ids_out) {
    cudaError_t e = cudaMemcpyAsync(ids_out, ws + L.ids, n * sizeof(int32_t),
                                    cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  if (w_out) {
    cudaError_t e =
        cudaMemcpyAsync(w_out, ws + L.w, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace beam
