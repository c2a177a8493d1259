// router.cu - FP32 router of the Beam MoE block ("Welcome Beam", section
// "Mixture of Experts": every expert is scored with a sigmoid; section
// "Residual Stream": the router is computed in FP32).
//
// Stage 0 (router_logits_kernel): logits = x W_r^T on CUDA cores in FP32,
// with an optional split over H so that small batches still fill the GPU.
// Partial sums are written per split and added in split order by stage 1, so
// the result does not depend on scheduling.
//
// Stage 1 (router_topk_kernel): one warp per token. Lane l holds PER
// consecutive experts; a group of E/G experts spans E/G/PER lanes. The warp
// computes the sigmoid scores, each group's sum of its two best choice
// scores, keeps the Gk best groups, picks the K best experts inside them
// (order key: value descending, expert id ascending) and the combine weights.
// The same CTA records, for its chunk of tokens, one bit per (expert, token)
// and the per-expert counts: the dispatch later derives every token's stable
// row inside its expert from these bits.
#include <math.h>

#include "internal.h"

namespace beam {
namespace {

constexpr int kRBM = 64;   // tokens per CTA
constexpr int kRBE = 128;  // experts per CTA
constexpr int kRBK = 32;   // K per shared-memory stage

__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const float* __restrict__ wr,
                                                            float* __restrict__ part, int T, int H,
                                                            int E, int kc) {
  __shared__ __align__(16) float xs[2][kRBK][kRBM];
  __shared__ __align__(16) float wsm[2][kRBK][kRBE];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.x * kRBM, e0 = blockIdx.y * kRBE;
  const int kbeg = blockIdx.z * kc;
  const int tx = tid & 15, ty = tid >> 4;  // experts {tx*4+q, 64+tx*4+q}, tokens ty*4+i

  // loader mapping: x rows tid&63, k offset (tid>>6)*8; w rows tid&127, k offset (tid>>7)*4+8r
  const int lx_t = m0 + (tid & 63), lx_k = (tid >> 6) * 8;
  const int lw_e = e0 + (tid & 127), lw_k = (tid >> 7) * 4;
  const bool x_ok = lx_t < T, w_ok = lw_e < E;
  const uint16_t* xrow = x + (size_t)(x_ok ? lx_t : 0) * H;
  const float* wrow = wr + (size_t)(w_ok ? lw_e : 0) * H;

  uint4 xr;
  float4 wv[4];
  auto load = [&](int k0) {
    xr = x_ok ? __ldg(reinterpret_cast<const uint4*>(xrow + k0 + lx_k)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int r = 0; r < 4; ++r)
      wv[r] = w_ok ? __ldg(reinterpret_cast<const float4*>(wrow + k0 + lw_k + 8 * r))
                   : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  auto store = [&](int buf) {
    const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xs[buf][lx_k + 2 * j][tid & 63] = __uint_as_float(xw[j] << 16);
      xs[buf][lx_k + 2 * j + 1][tid & 63] = __uint_as_float(xw[j] & 0xFFFF0000u);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      wsm[buf][lw_k + 8 * r + 0][tid & 127] = wv[r].x;
      wsm[buf][lw_k + 8 * r + 1][tid & 127] = wv[r].y;
      wsm[buf][lw_k + 8 * r + 2][tid & 127] = wv[r].z;
      wsm[buf][lw_k + 8 * r + 3][tid & 127] = wv[r].w;
    }
  };

  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = kc / kRBK;
  load(kbeg);
  store(0);
  __syncthreads();
  for (int it = 0; it < nk; ++it) {
    const int buf = it & 1;
    if (it + 1 < nk) load(kbeg + (it + 1) * kRBK);
#pragma unroll
    for (int k = 0; k < kRBK; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[buf][k][ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&wsm[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&wsm[buf][k][64 + tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (it + 1 < nk) store(buf ^ 1);
    __syncthreads();
  }

  float* out = part + (size_t)blockIdx.z * T * E;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = m0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int e = e0 + h * 64 + tx * 4;
      if ((E & 3) == 0 && e + 3 < E) {
        *reinterpret_cast<float4*>(out + (size_t)t * E + e) =
            make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
      } else {
        for (int q = 0; q < 4; ++q)
          if (e + q < E) out[(size_t)t * E + e + q] = acc[i][4 * h + q];
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
  const float* part;  // [split_k][T][E] partial logits, or NULL (ids given)
  int split_k;
  const float* bias;  // [E] or NULL
  int bias_mode;
  int T, E, G, Gk, K, renorm;
  float scale;
  int32_t* ids;        // [T][K]
  float* w;            // [T][K]
  int32_t* chunk_cnt;  // [nchunks][E]
  uint32_t* chunk_mask;// [nchunks][E][kChunkWords]
};

template <int PER>
__global__ void __launch_bounds__(256) router_topk_kernel(TopkArgs a) {
  __shared__ uint32_t smask[512 * kChunkWords];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = blockIdx.x, t0 = c * kChunk;
  const int E = a.E, K = a.K;
  for (int i = tid; i < E * kChunkWords; i += 256) smask[i] = 0u;
  __syncthreads();

  const int gs = E / a.G;          // experts per group
  const int lg = gs / PER;         // lanes per group (power of two)
  const bool active = lane * PER < E;
  const int gid = active ? (lane * PER) / gs : 0x7fffffff;

  for (int tl = warp; tl < kChunk; tl += 8) {
    const int t = t0 + tl;
    if (t >= a.T) break;
    float s[PER], ch[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = lane * PER + j;
      s[j] = 0.f;
      ch[j] = -INFINITY;
      if (e < E) {
        float l = 0.f;
        for (int sp = 0; sp < a.split_k; ++sp) l += a.part[((size_t)sp * a.T + t) * E + e];
        const float b = a.bias ? a.bias[e] : 0.f;
        if (a.bias_mode == 0) l += b;
        s[j] = 1.0f / (1.0f + expf(-l));
        ch[j] = a.bias_mode == 1 ? s[j] + b : s[j];
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
          if (e < E && !((taken >> j) & 1u) && (ch[j] > bv || (ch[j] == bv && e < be))) {
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
      atomicOr(&smask[my_e * kChunkWords + (tl >> 5)], 1u << (tl & 31));
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += 256) {
    int cnt = 0;
#pragma unroll
    for (int wd = 0; wd < kChunkWords; ++wd) {
      const uint32_t m = smask[e * kChunkWords + wd];
      cnt += __popc(m);
      a.chunk_mask[((size_t)c * E + e) * kChunkWords + wd] = m;
    }
    a.chunk_cnt[(size_t)c * E + e] = cnt;
  }
}

// Caller-supplied routes: copy ids / weights into the workspace and record the
// chunk bits and counts. Out-of-range ids are dropped (id -1) and flagged.
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
  for (int e = tid; e < E; e += 256) {
    int cnt = 0;
#pragma unroll
    for (int wd = 0; wd < kChunkWords; ++wd) {
      const uint32_t m = smask[e * kChunkWords + wd];
      cnt += __popc(m);
      a.chunk_mask[((size_t)c * E + e) * kChunkWords + wd] = m;
    }
    a.chunk_cnt[(size_t)c * E + e] = cnt;
  }
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
  a.chunk_cnt = reinterpret_cast<int32_t*>(ws + L.chunk_cnt);
  a.chunk_mask = reinterpret_cast<uint32_t*>(ws + L.chunk_mask);
  return a;
}

}  // namespace

int router_split_k(int64_t T, int H, int E, int sms) {
  const int64_t tiles = ((T + kRBM - 1) / kRBM) * ((E + kRBE - 1) / kRBE);
  const int max_split = H / kRBK;
  int want = (int)((2 * (int64_t)sms + tiles - 1) / tiles);
  if (want < 1) want = 1;
  int best = 1;
  for (int s = 1; s <= max_split; ++s)
    if (max_split % s == 0 && s <= want) best = s;
  return best;
}

cudaError_t launch_router_logits(const beam_moe_cfg& c, const Layout& L, const uint16_t* x,
                                 const float* w_router, char* ws, cudaStream_t st) {
  const int H = c.hidden, E = c.n_experts;
  dim3 grid((unsigned)((L.T + kRBM - 1) / kRBM), (unsigned)((E + kRBE - 1) / kRBE),
            (unsigned)L.split_k);
  router_logits_kernel<<<grid, 256, 0, st>>>(x, w_router, reinterpret_cast<float*>(ws + L.logits),
                                              (int)L.T, H, E, H / L.split_k);
  return cudaGetLastError();
}

cudaError_t launch_router_topk(const beam_moe_cfg& c, const Layout& L, const float* bias,
                               char* ws, cudaStream_t st) {
  TopkArgs a = topk_args(c, L, ws);
  a.bias = bias;
  const int E = c.n_experts;
  const dim3 grid((unsigned)L.nchunks);
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
