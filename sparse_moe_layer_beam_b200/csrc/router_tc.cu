// router_tc.cu - the router GEMM of the Beam MoE block on tensor cores, in
// FP32 arithmetic ("Welcome Beam", section "Residual Stream": the router is
// computed in FP32; section "Mixture of Experts": every expert is scored).
//
// The FP32 router weights are split exactly into three bf16 planes,
// w = w1 + w2 + w3: w1 = bf16(w), w2 = bf16(w - w1), w3 = w - w1 - w2. An FP32
// significand has 24 bits and each rounding peels off the next 8, so the
// third remainder fits a bf16 exactly. x is bf16, so every product x * w_i is
// exact in FP32, and the tensor core accumulates the 3 H products of a logit
// in FP32 in TMEM. That is the same FP32 contraction the CUDA-core kernel in
// router.cu computes, reordered.
//
// Kernel layout: swap-AB like the expert GEMMs. A tile is 128 experts (MMA M)
// x BN tokens (MMA N); each K step of 64 loads the three planes' 128 x 64
// weight tiles and one BN x 64 token tile, and issues 3 x 4 MMAs into one
// accumulator. Warp 0 is the TMA producer, warp 1 the MMA issuer, warps 2-5
// the epilogue (one TMEM lane quarter each); the accumulator is
// double-buffered. For small batches the K range is split over CTAs; every
// split writes its own slice of partial logits [split][T][E], which the
// top-k stage adds in split order, exactly as for the CUDA-core kernel.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace beam {
namespace {

constexpr int kRK = 64;          // K per pipeline stage (128 bytes of bf16)
constexpr int kRThreads = 192;
constexpr int kRPlaneBytes = kTileM * kRK * 2;  // one plane's 128 x 64 tile
constexpr int kMaxTcSplit = 16;  // bounds the partial logits the top-k stage reads

struct RouterTcParams {
  float* part;   // [n_split][T][E] partial logits
  int T, E;
  int nkb;       // K blocks (H / 64)
  int kper;      // K blocks per split
  int n_split, n_nt, n_mb;
  unsigned* status;
};

template <int BN>
struct RCfg {
  static constexpr int kBBytes = BN * kRK * 2;
  static constexpr int kStageBytes = 3 * kRPlaneBytes + kBBytes;
  static constexpr int kStagesRaw = (220 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 6 ? 6 : kStagesRaw;
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
  static_assert(kStages >= 2, "pipeline too shallow");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// tile -> (split, token tile, expert block); the expert block is fastest, so
// the CTAs reading the same token tile run together and share it in L2
__device__ __forceinline__ void decode_rtile(int tile, const RouterTcParams& p, int& s, int& nt,
                                             int& mb) {
  mb = tile % p.n_mb;
  const int rest = tile / p.n_mb;
  nt = rest % p.n_nt;
  s = rest / p.n_nt;
}

__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ wr,
                                                           uint16_t* __restrict__ w3, int64_t n,
                                                           uint32_t* __restrict__ bits,
                                                           int64_t n_bits_words) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float w = wr[i];
    const __nv_bfloat16 b1 = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(b1);  // exact
    const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(b2);  // exact, at most 8 significant bits
    w3[i] = __bfloat16_as_ushort(b1);
    w3[n + i] = __bfloat16_as_ushort(b2);
    w3[2 * n + i] = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
  }
  // clear the dispatch bits that the top-k stage sets
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_bits_words; i += stride)
    bits[i] = 0u;
}

template <int BN>
__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_x, const RouterTcParams p) {
  using C = RCfg<BN>;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // stage: [plane 0][plane 1][plane 2][tokens]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = p.n_split * p.n_nt * p.n_mb;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint64_t pol = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int s, nt, mb;
        decode_rtile(tile, p, s, nt, mb);
        const int kb0 = s * p.kper, kb1 = min(p.nkb, kb0 + p.kper);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          for (int pl = 0; pl < 3; ++pl)
            tma_load_2d(sa + pl * kRPlaneBytes, &tm_w, &full[stage], kb * kRK,
                        pl * p.E + mb * kTileM, pol);
          tma_load_2d(sa + 3 * kRPlaneBytes, &tm_x, &full[stage], kb * kRK, nt * BN, pol);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t i = first; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), nullptr, nullptr, 0u,
                  100000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kTileM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int s, nt, mb;
        decode_rtile(tile, p, s, nt, mb);
        const int kb0 = s * p.kper, kb1 = min(p.nkb, kb0 + p.kper);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, kFlagMma)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint64_t db = smem_desc_k_sw128(sa + 3 * kRPlaneBytes);
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {
            const uint64_t da = smem_desc_k_sw128(sa + pl * kRPlaneBytes);
#pragma unroll
            for (int k4 = 0; k4 < kRK / 16; ++k4)
              umma_bf16(d, da + 2u * k4, db + 2u * k4, idesc, (kb != kb0) | pl | k4);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    // lane quarter q holds experts mb*128 + 32q .. +31; column j is token
    // nt*BN + j; a warp's store of one token is 32 consecutive floats
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int s, nt, mb;
      decode_rtile(tile, p, s, nt, mb);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, kFlagEpilogue)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int e = mb * kTileM + q * 32 + lane;
      const int t0 = nt * BN;
      float* out = p.part + ((size_t)s * p.T + t0) * p.E + e;
      const int n_tok = min(BN, p.T - t0);
      for (int c0 = 0; c0 < n_tok; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tb + c0, v);
        tmem_ld_wait();
        if (e < p.E) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n_tok) out[(size_t)(c0 + j) * p.E] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <int BN>
cudaError_t run_router_tc(const CUtensorMap& tw, const CUtensorMap& tx, const RouterTcParams& p,
                          cudaStream_t st) {
  using C = RCfg<BN>;
  static PerDevice configured;  // the shared-memory attribute, once per device
  int unused = 0;
  cudaError_t err = per_device(configured, &unused, [](int*) {
    return cudaFuncSetAttribute(router_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  const int total = p.n_split * p.n_nt * p.n_mb;
  const int grid = total < device_sm_count() ? total : device_sm_count();
  router_tc_kernel<BN><<<grid, kRThreads, C::kSmemBytes, st>>>(tw, tx, p);
  return cudaGetLastError();
}

}  // namespace

bool router_tc_supported(const beam_moe_cfg& c) { return c.hidden % kRK == 0; }

int router_tc_bn(int64_t T) { return T <= 64 ? 64 : (T <= 128 ? 128 : 256); }

// K blocks per split: minimises waves x (K blocks per CTA + a fixed cost of
// two K blocks per tile); ties go to fewer splits.
int router_tc_kper(int64_t T, int H, int E, int sms) {
  const int nkb = H / kRK;
  const int bn = router_tc_bn(T);
  const int min_kper = (nkb + kMaxTcSplit - 1) / kMaxTcSplit;
  const int64_t tiles = ((T + bn - 1) / bn) * ((E + kTileM - 1) / kTileM);
  const int64_t slots = sms > 0 ? sms : 1;
  int best = nkb;
  double best_cost = 1e30;
  for (int kper = nkb; kper >= min_kper; --kper) {
    const int64_t splits = (nkb + kper - 1) / kper;
    if ((splits - 1) * kper >= nkb) continue;  // an empty split
    const int64_t waves = (tiles * splits + slots - 1) / slots;
    const double cost = (double)waves * (kper + 2);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = kper;
    }
  }
  return best;
}

cudaError_t launch_router_tc(const beam_moe_cfg& c, const Layout& L, const uint16_t* x,
                             const float* w_router, char* ws, cudaStream_t st) {
  const int H = c.hidden, E = c.n_experts;
  uint16_t* w3 = reinterpret_cast<uint16_t*>(ws + L.w3);
  const int64_t n = (int64_t)E * H;
  const int64_t nbits = (int64_t)L.nchunks * E * kChunkWords;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4L * device_sm_count()) blocks = 4L * device_sm_count();
  router_split_kernel<<<(unsigned)blocks, 256, 0, st>>>(
      w_router, w3, n, reinterpret_cast<uint32_t*>(ws + L.chunk_mask), nbits);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  const int bn = router_tc_bn(L.T);
  CUtensorMap tw, tx;
  err = encode_tmap_2d_bf16(&tw, w3, (uint64_t)H, (uint64_t)3 * E, kRK, kTileM);
  if (err != cudaSuccess) return err;
  err = encode_tmap_2d_bf16(&tx, x, (uint64_t)H, (uint64_t)L.T, kRK, (uint32_t)bn);
  if (err != cudaSuccess) return err;
  RouterTcParams p;
  p.part = reinterpret_cast<float*>(ws + L.logits);
  p.T = (int)L.T;
  p.E = E;
  p.nkb = H / kRK;
  p.kper = L.router_kper;
  p.n_split = L.split_k;
  p.n_nt = (int)((L.T + bn - 1) / bn);
  p.n_mb = (E + kTileM - 1) / kTileM;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);
  if (bn == 64) return run_router_tc<64>(tw, tx, p, st);
  if (bn == 128) return run_router_tc<128>(tw, tx, p, st);
  return run_router_tc<256>(tw, tx, p, st);
}

}  // namespace beam
