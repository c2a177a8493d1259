// dispatch.cu - token dispatch and combine of the Beam MoE block.
//
// The pages describe routing and combining ("Welcome Beam", section "Mixture
// of Experts": only 8 experts run per token; their outputs are combined with
// normalized weights and scaled by 2.5); grouping rows by expert so that every
// expert runs as one dense GEMM is this library's design.
//
//   scan     per-expert counts, first row of each expert (exclusive scan),
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

__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ chunk_cnt, int nchunks,
                                                    int E, int bn, int32_t* __restrict__ counts,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ nb_off,
                                                    int32_t* __restrict__ counts_out) {
  __shared__ int32_t part[1024];
  __shared__ int32_t s_off[513];
  __shared__ int32_t s_nb[513];
  const int tid = threadIdx.x;
  const int tpe = 1024 / E;  // threads per expert (E <= 512)
  const int e = tid % E, j = tid / E;
  const bool act = j < tpe;
  const int L = (nchunks + tpe - 1) / tpe;
  const int c0 = j * L, c1 = min(nchunks, c0 + L);
  int sum = 0;
  if (act)
    for (int c = c0; c < c1; ++c) sum += chunk_cnt[(size_t)c * E + e];
  part[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int run = 0, nrun = 0;
    for (int x = 0; x < E; ++x) {
      int tot = 0;
      for (int q = 0; q < tpe; ++q) tot += part[q * E + x];
      s_off[x] = run;
      s_nb[x] = nrun;
      run += tot;
      nrun += (tot + bn - 1) / bn;
    }
    s_off[E] = run;
    s_nb[E] = nrun;
  }
  __syncthreads();
  if (act) {
    int run = s_off[e];
    for (int q = 0; q < j; ++q) run += part[q * E + e];
    for (int c = c0; c < c1; ++c) {
      const size_t i = (size_t)c * E + e;
      const int v = chunk_cnt[i];
      chunk_cnt[i] = run;
      run += v;
    }
  }
  for (int x = tid; x <= E; x += 1024) {
    offsets[x] = s_off[x];
    nb_off[x] = s_nb[x];
    if (x < E) {
      counts[x] = s_off[x + 1] - s_off[x];
      if (counts_out) counts_out[x] = s_off[x + 1] - s_off[x];
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
    pos[(size_t)t * K + tid] = p;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  const int nv = H / 8;
  for (int v = tid; v < nv; v += 128) {
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
  for (int v = tid; v < nv; v += 128) {
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
  scan_kernel<<<1, 1024, 0, st>>>(reinterpret_cast<int32_t*>(ws + L.chunk_cnt), L.nchunks,
                                  c.n_experts, L.bn, reinterpret_cast<int32_t*>(ws + L.counts),
                                  reinterpret_cast<int32_t*>(ws + L.offsets),
                                  reinterpret_cast<int32_t*>(ws + L.nb_off), counts_out);
  return cudaGetLastError();
}

cudaError_t launch_permute(const beam_moe_cfg& c, const Layout& L, const uint16_t* x, char* ws,
                           cudaStream_t st) {
  permute_kernel<<<(unsigned)L.T, 128, 0, st>>>(
      x, c.hidden, c.top_k, c.n_experts, reinterpret_cast<const int32_t*>(ws + L.ids),
      reinterpret_cast<const int32_t*>(ws + L.chunk_cnt),
      reinterpret_cast<const uint32_t*>(ws + L.chunk_mask), reinterpret_cast<int32_t*>(ws + L.pos),
      reinterpret_cast<uint16_t*>(ws + L.xp));
  return cudaGetLastError();
}

cudaError_t launch_combine(const beam_moe_cfg& c, const Layout& L, uint16_t* out, char* ws,
                           cudaStream_t st) {
  combine_kernel<<<(unsigned)L.T, 128, 0, st>>>(
      reinterpret_cast<const float*>(ws + L.xp), c.hidden, c.top_k,
      reinterpret_cast<const int32_t*>(ws + L.pos), reinterpret_cast<const float*>(ws + L.w), out);
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
