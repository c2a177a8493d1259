// router.cu - FP32 router of the Beam MoE block ("Welcome Beam", section
// "Mixture of Experts": every expert is scored with a sigmoid; section
// "Residual Stream": the router is computed in FP32).
//
// Stage 0 (router_logits_kernel): logits = x W_r^T on CUDA cores in FP32,
// 128 tokens x 128 experts per CTA, 8 x 8 per thread as paired FP32 FMAs
// (fma.rn.f32x2), 32 k per shared-memory stage, with an optional split over H
// (at most 16 parts) so that small batches still fill the GPU. Each logit is
// a chain of FP32 FMAs in ascending k inside its split; partial sums are
// written per split and added in split order by stage 1, so the result does
// not depend on scheduling. The same kernel clears the dispatch bits that
// stage 1 sets.
//
// Stage 1 (router_topk_kernel): one warp per token. Lane l holds PER
// consecutive experts; a group of E/G experts spans E/G/PER lanes. The warp
// computes the sigmoid scores, each group's sum of its two best choice
// scores, keeps the Gk best groups, picks the K best experts inside them
// (order key: value descending, expert id ascending) and the combine weights,
// and sets one bit per (expert, token) in its 128-token chunk (an OR, so the
// result does not depend on the order of the warps). The dispatch derives
// every token's stable row inside its expert from these bits.
#include <math.h>

#include "internal.h"

namespace beam {
namespace {

constexpr int kRBM = 128;  // tokens per CTA
constexpr int kRBE = 128;  // experts per CTA
constexpr int kRBK = 32;   // K per shared-memory stage
constexpr int kMaxSplit = 16;
constexpr int kRawLd = kRBK + 4;  // row stride of the raw W_r stage (16-byte chunks spread over banks)
// [2 stages][x, w][kRBK][128] fp32, then the raw W_r stage [128][kRawLd] fp32
constexpr int kRouterSmem = (2 * 2 * kRBK * kRBM + kRBE * kRawLd) * 4;

// d = a * b + c on two FP32 lanes at once (fma.rn.f32x2: each lane is an
// ordinary round-to-nearest FP32 FMA, so results equal two fmaf calls). Half
// the FMA instructions of the scalar loop for the same arithmetic.
__device__ __forceinline__ void fma2(unsigned long long& d, unsigned long long a,
                                     unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

__device__ __forceinline__ unsigned long long splat2(float v) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
  return r;
}

// 16-byte asynchronous copy global -> shared (zero-filled when src_bytes is
// 0), and the wait for every copy this thread has issued.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(src_bytes)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

__global__ void __launch_bounds__(256, 2) router_logits_kernel(const uint16_t* __restrict__ x,
                                                               const float* __restrict__ wr,
                                                               float* __restrict__ part, int T,
                                                               int H, int E, int kc,
                                                               uint32_t* __restrict__ bits,
                                                               int64_t n_bits_words) {
  extern __shared__ __align__(16) float rsm[];
  float (*xs)[kRBK][kRBM] = reinterpret_cast<float (*)[kRBK][kRBM]>(rsm);
  float (*wsm)[kRBK][kRBE] = reinterpret_cast<float (*)[kRBK][kRBE]>(rsm + 2 * kRBK * kRBM);
  float (*raw)[kRawLd] = reinterpret_cast<float (*)[kRawLd]>(rsm + 4 * kRBK * kRBM);
  const int tid = threadIdx.x;
  {  // clear the dispatch bits set by stage 1
    const int64_t nthreads = (int64_t)gridDim.x * gridDim.y * gridDim.z * blockDim.x;
    const int64_t cta = ((int64_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    for (int64_t i = cta * blockDim.x + tid; i < n_bits_words; i += nthreads) bits[i] = 0u;
  }
  const int m0 = blockIdx.x * kRBM, e0 = blockIdx.y * kRBE;
  const int kbeg = blockIdx.z * kc;
  // compute mapping: tokens {ty*4+i, 64+ty*4+i}, experts {tx*4+j, 64+tx*4+j}
  const int tx = tid & 15, ty = tid >> 4;
  // loader mapping: row tid&127 (a token of x, an expert of W_r), k offset
  // (tid>>7)*16 inside the stage: 16 consecutive k of one row per thread
  const int lrow = tid & 127, lk = (tid >> 7) * 16;
  const bool x_ok = m0 + lrow < T, w_ok = e0 + lrow < E;
  const uint16_t* xrow = x + (size_t)(x_ok ? m0 + lrow : 0) * H;
  const float* wrow = wr + (size_t)(w_ok ? e0 + lrow : 0) * H;

  // x goes through registers (bf16 -> fp32 on the way into shared memory).
  // W_r, already fp32, is copied asynchronously one stage ahead into a raw
  // row-major stage; each thread then moves the cells it copied itself into
  // their transposed place, so no register holds W_r across the compute.
  uint4 xr[2];
  auto load_x = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 2; ++q)
      xr[q] = x_ok ? __ldg(reinterpret_cast<const uint4*>(xrow + k0 + lk + 8 * q))
                   : make_uint4(0, 0, 0, 0);
  };
  auto store_x = [&](int buf) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t xw[4] = {xr[q].x, xr[q].y, xr[q].z, xr[q].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // bf16 -> fp32 is exact: the bits move up 16
        xs[buf][lk + 8 * q + 2 * j][lrow] = __uint_as_float(xw[j] << 16);
        xs[buf][lk + 8 * q + 2 * j + 1][lrow] = __uint_as_float(xw[j] & 0xFFFF0000u);
      }
    }
  };
  auto copy_w = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      cp_async16(&raw[lrow][lk + 4 * q], wrow + k0 + lk + 4 * q, w_ok ? 16u : 0u);
    cp_async_commit();
  };
  auto store_w = [&](int buf) {
    cp_async_wait_all();  // this thread's own copies: no barrier needed to read them
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(&raw[lrow][lk + 4 * q]);
      wsm[buf][lk + 4 * q + 0][lrow] = v.x;
      wsm[buf][lk + 4 * q + 1][lrow] = v.y;
      wsm[buf][lk + 4 * q + 2][lrow] = v.z;
      wsm[buf][lk + 4 * q + 3][lrow] = v.w;
    }
  };

  // acc[i][jj] holds experts (2 jj, 2 jj + 1) of this thread's 8 for token i
  unsigned long long acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;

  const int nk = kc / kRBK;
  load_x(kbeg);
  copy_w(kbeg);
  store_x(0);
  store_w(0);
  __syncthreads();
  for (int it = 0; it < nk; ++it) {
    const int buf = it & 1;
    if (it + 1 < nk) {
      load_x(kbeg + (it + 1) * kRBK);
      copy_w(kbeg + (it + 1) * kRBK);
    }
#pragma unroll
    for (int k = 0; k < kRBK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[buf][k][64 + ty * 4]);
      const ulonglong2 b0 = *reinterpret_cast<const ulonglong2*>(&wsm[buf][k][tx * 4]);
      const ulonglong2 b1 = *reinterpret_cast<const ulonglong2*>(&wsm[buf][k][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const unsigned long long bv[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const unsigned long long a2 = splat2(av[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) fma2(acc[i][j], a2, bv[j]);
      }
    }
    if (it + 1 < nk) {
      store_x(buf ^ 1);
      store_w(buf ^ 1);
    }
    __syncthreads();
  }

  float* out = part + (size_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + (i >> 2) * 64 + ty * 4 + (i & 3);
    if (t >= T) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float v[4];
      asm("mov.b64 {%0, %1}, %2;" : "=f"(v[0]), "=f"(v[1]) : "l"(acc[i][2 * h]));
      asm("mov.b64 {%0, %1}, %2;" : "=f"(v[2]), "=f"(v[3]) : "l"(acc[i][2 * h + 1]));
      const int e = e0 + h * 64 + tx * 4;
      if ((E & 3) == 0 && e + 3 < E) {
        *reinterpret_cast<float4*>(out + (size_t)t * E + e) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
        for (int q = 0; q < 4; ++q)
          if (e + q < E) out[(size_t)t * E + e + q] = v[q];
      }
    }
  }
}

// Warp argmax with key (value descending, index ascending), carrying `s`.
__device__ __forceinline__ void warp_argmax(float& v, int& idx, float& s) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
    const float os = __shfl_xor_sync(0xffffffffu, s, off);
    if (ov > v || (ov == v && oi < idx)) {
      v = ov;
      idx = oi;
      s = os;
    }
  }
}

struct TopkArgs {
  const float* part;  // [split_k][T][E] partial logits
  int split_k;
  const float* bias;  // [E] or NULL
  int bias_mode;
  int T, E, G, Gk, K, renorm;
  float scale;
  int32_t* ids;         // [T][K]
  float* w;             // [T][K]
  uint32_t* chunk_mask; // [nchunks][E][kChunkWords]
};

// Sum of the split partial logits of PER consecutive experts, split order.
template <int PER>
__device__ __forceinline__ void load_logits(const float* __restrict__ p, size_t stride, int n,
                                            float (&l)[PER]) {
#pragma unroll
  for (int j = 0; j < PER; ++j) l[j] = 0.f;
  if constexpr (PER % 4 == 0) {
#pragma unroll 4
    for (int sp = 0; sp < n; ++sp) {
      const float4* q = reinterpret_cast<const float4*>(p + sp * stride);
#pragma unroll
      for (int v = 0; v < PER / 4; ++v) {
        const float4 f = __ldg(q + v);
        l[4 * v] += f.x;
        l[4 * v + 1] += f.y;
        l[4 * v + 2] += f.z;
        l[4 * v + 3] += f.w;
      }
    }
  } else {
    for (int sp = 0; sp < n; ++sp)
#pragma unroll
      for (int j = 0; j < PER; ++j) l[j] += __ldg(p + sp * stride + j);
  }
}

template <int PER>
__global__ void __launch_bounds__(256) router_topk_kernel(TopkArgs a) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int t = blockIdx.x * 8 + (tid >> 5);
  if (t >= a.T) return;  // whole warps leave together
  const int E = a.E, K = a.K;
  const int gs = E / a.G;   // experts per group
  const int lg = gs / PER;  // lanes per group (power of two)
  const bool active = lane * PER < E;
  const int gid = active ? (lane * PER) / gs : 0x7fffffff;

  float s[PER], ch[PER];
  if (active) {
    float l[PER];
    load_logits<PER>(a.part + (size_t)t * E + lane * PER, (size_t)a.T * E, a.split_k, l);
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      const float b = a.bias ? a.bias[e] : 0.f;
      const float lj = a.bias_mode == 0 ? l[j] + b : l[j];
      s[j] = 1.0f / (1.0f + expf(-lj));
      ch[j] = a.bias_mode == 1 ? s[j] + b : s[j];
    }
  } else {
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      s[j] = 0.f;
      ch[j] = -INFINITY;
    }
  }
  // group score: sum of the two best choice scores of the group
  float b1 = -INFINITY, b2 = -INFINITY;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (ch[j] > b1) {
      b2 = b1;
      b1 = ch[j];
    } else if (ch[j] > b2) {
      b2 = ch[j];
    }
  }
  for (int off = 1; off < lg; off <<= 1) {
    const float o1 = __shfl_xor_sync(0xffffffffu, b1, off);
    const float o2 = __shfl_xor_sync(0xffffffffu, b2, off);
    const float n2 = fmaxf(fminf(b1, o1), fmaxf(b2, o2));
    b1 = fmaxf(b1, o1);
    b2 = n2;
  }
  const float gscore = b1 + b2;
  // keep the Gk best groups
  bool kept = false;
  for (int r = 0; r < a.Gk; ++r) {
    float v = (active && !kept) ? gscore : -INFINITY;
    int id = gid;
    float unused = 0.f;
    warp_argmax(v, id, unused);
    if (gid == id) kept = true;
  }
  // top-K experts inside the kept groups
  uint32_t taken = 0u;
  int my_e = -1;
  float my_s = 0.f, wsum = 0.f;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY, bs = 0.f;
    int be = 0x7fffffff;
    if (kept) {
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = lane * PER + j;
        if (!((taken >> j) & 1u) && (ch[j] > bv || (ch[j] == bv && e < be))) {
          bv = ch[j];
          be = e;
          bs = s[j];
        }
      }
    }
    warp_argmax(bv, be, bs);
    if (lane == be / PER) taken |= 1u << (be - lane * PER);
    if (lane == k) {
      my_e = be;
      my_s = bs;
    }
    wsum += bs;
  }
  if (lane < K) {
    const float wk = a.renorm ? my_s / wsum : my_s;
    a.ids[(size_t)t * K + lane] = my_e;
    a.w[(size_t)t * K + lane] = a.scale * wk;
    const int c = t / kChunk, tl = t - c * kChunk;
    atomicOr(&a.chunk_mask[((size_t)c * E + my_e) * kChunkWords + (tl >> 5)], 1u << (tl & 31));
  }
}

// Caller-supplied routes: copy ids / weights into the workspace and write the
// chunk bits. Out-of-range ids are dropped (id -1) and flagged.
__global__ void __launch_bounds__(256) routes_given_kernel(const int32_t* __restrict__ ids_in,
                                                           const float* __restrict__ w_in,
                                                           TopkArgs a, unsigned* status) {
  __shared__ uint32_t smask[512 * kChunkWords];
  const int tid = threadIdx.x;
  const int c = blockIdx.x, t0 = c * kChunk;
  const int E = a.E, K = a.K;
  for (int i = tid; i < E * kChunkWords; i += 256) smask[i] = 0u;
  __syncthreads();
  for (int i = tid; i < kChunk * K; i += 256) {
    const int tl = i / K, t = t0 + tl;
    if (t >= a.T) break;
    const size_t o = (size_t)t * K + (i - tl * K);
    int e = ids_in[o];
    if (e < 0 || e >= E) {
      atomicOr(status, kFlagBadExpert);
      e = -1;
    } else {
      atomicOr(&smask[e * kChunkWords + (tl >> 5)], 1u << (tl & 31));
    }
    a.ids[o] = e;
    a.w[o] = w_in[o];
  }
  __syncthreads();
  for (int i = tid; i < E * kChunkWords; i += 256)
    a.chunk_mask[(size_t)c * E * kChunkWords + i] = smask[i];
}

TopkArgs topk_args(const beam_moe_cfg& c, const Layout& L, char* ws) {
  TopkArgs a;
  a.part = reinterpret_cast<const float*>(ws + L.logits);
  a.split_k = L.split_k;
  a.bias = nullptr;
  a.bias_mode = c.bias_mode;
  a.T = (int)L.T;
  a.E = c.n_experts;
  a.G = c.n_group;
  a.Gk = c.topk_group;
  a.K = c.top_k;
  a.renorm = c.renormalize;
  a.scale = c.routed_scale;
  a.ids = reinterpret_cast<int32_t*>(ws + L.ids);
  a.w = reinterpret_cast<float*>(ws + L.w);
  a.chunk_mask = reinterpret_cast<uint32_t*>(ws + L.chunk_mask);
  return a;
}

}  // namespace

// Split of H for the router GEMM: the divisor of H/16 (at most 16) that
// minimises waves x work per CTA, with two CTAs resident per SM; ties go to
// the smaller split (fewer partial sums for stage 1 to read).
int router_split_k(int64_t T, int H, int E, int sms) {
  const int64_t tiles = ((T + kRBM - 1) / kRBM) * ((E + kRBE - 1) / kRBE);
  const int64_t slots = 2 * (int64_t)(sms > 0 ? sms : 1);
  const int max_split = H / kRBK;
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= max_split && s <= kMaxSplit; ++s) {
    if (max_split % s != 0) continue;
    const int64_t waves = (tiles * s + slots - 1) / slots;
    const double cost = (double)waves / s;
    if (cost < best_cost - 1e-12) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_router_logits(const beam_moe_cfg& c, const Layout& L, const uint16_t* x,
                                 const float* w_router, char* ws, cudaStream_t st) {
  if (L.router_tc) return launch_router_tc(c, L, x, w_router, ws, st);
  const int H = c.hidden, E = c.n_experts;
  static PerDevice configured;  // the shared-memory attribute, once per device
  int unused = 0;
  cudaError_t err = per_device(configured, &unused, [](int*) {
    return cudaFuncSetAttribute(router_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kRouterSmem);
  });
  if (err != cudaSuccess) return err;
  dim3 grid((unsigned)((L.T + kRBM - 1) / kRBM), (unsigned)((E + kRBE - 1) / kRBE),
            (unsigned)L.split_k);
  router_logits_kernel<<<grid, 256, kRouterSmem, st>>>(
      x, w_router, reinterpret_cast<float*>(ws + L.logits), (int)L.T, H, E, H / L.split_k,
      reinterpret_cast<uint32_t*>(ws + L.chunk_mask), (int64_t)L.nchunks * E * kChunkWords);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const beam_moe_cfg& c, const Layout& L, const float* bias,
                               char* ws, cudaStream_t st) {
  TopkArgs a = topk_args(c, L, ws);
  a.bias = bias;
  const int E = c.n_experts;
  const dim3 grid((unsigned)((L.T + 7) / 8));
  if (E <= 32) router_topk_kernel<1><<<grid, 256, 0, st>>>(a);
  else if (E <= 64) router_topk_kernel<2><<<grid, 256, 0, st>>>(a);
  else if (E <= 128) router_topk_kernel<4><<<grid, 256, 0, st>>>(a);
  else if (E <= 256) router_topk_kernel<8><<<grid, 256, 0, st>>>(a);
  else router_topk_kernel<16><<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_routes_given(const beam_moe_cfg& c, const Layout& L, const int32_t* ids,
                                const float* w, char* ws, cudaStream_t st) {
  TopkArgs a = topk_args(c, L, ws);
  routes_given_kernel<<<(unsigned)L.nchunks, 256, 0, st>>>(
      ids, w, a, reinterpret_cast<unsigned*>(ws + L.status));
  return cudaGetLastError();
}

}  // namespace beam
