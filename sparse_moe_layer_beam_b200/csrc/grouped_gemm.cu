// grouped_gemm.cu - the two expert GEMMs of the Beam MoE block on 5th-generation
// tensor cores ("Welcome Beam", section "Mixture of Experts": each expert is a
// SwiGLU MLP, hidden 5120, intermediate 2560; section "Residual Stream": the
// SwiGLU product is computed in FP32).
//
//   gate/up:  [g | u] = W13_e x   for every row routed to expert e,
//             h = silu(g) * u in FP32, stored bf16          (K = H)
//   down:     y = W2_e h, stored fp32                         (K = I)
//
// Design (sm_100a):
//  - Swap-AB: 128 weight rows are the MMA M dimension and the routed tokens of
//    one expert are N (a multiple of 16, at most BN). At decode an expert sees
//    a handful of tokens, so the weights stream through the M side at full
//    tile efficiency; at large T the tokens fill N up to 256.
//  - One persistent CTA per SM walks a static tile list (expert, weight
//    block, token block) built on the device from the routed counts: tile i
//    of expert e covers weight block i / nblk_e and token block i % nblk_e, so
//    consecutive tiles share weights through L2.
//  - Warp 0 (one thread) issues TMA loads of the weight tile(s) and the token
//    tile into a STAGES-deep shared-memory ring (128-byte swizzle, 64 K per
//    stage); warp 1 (one thread) issues tcgen05.mma into TMEM accumulators
//    (two per tile for gate/up: gate and up of the same 128 intermediate
//    rows); warps 2-5 read TMEM (tcgen05.ld), apply the epilogue and store.
//    Accumulators are double-buffered in TMEM when they fit in 512 columns.
//  - Every wait is bounded; a timeout sets a status bit and the CTA unwinds
//    after its own copies and MMAs have completed.
#include <cuda_bf16.h>

#include "grouped_gemm.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace beam {
namespace {

using gg::GemmParams;
using gg::decode_tile;
using gg::pow2_at_least;
using gg::silu_mul;


constexpr int kThreads = 192;

template <bool GATEUP, int BN>
struct Cfg {
  static constexpr int kABytes = kTileM * kTileK * 2;
  static constexpr int kNA = GATEUP ? 2 : 1;
  static constexpr int kBBytes = BN * kTileK * 2;
  static constexpr int kStageBytes = kNA * kABytes + kBBytes;
  static constexpr int kStagesRaw = (220 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kAccCols = GATEUP ? 2 * BN : BN;
  static constexpr int kAccStages = (2 * kAccCols <= 512) ? 2 : 1;
  static constexpr int kTmemCols = pow2_at_least(kAccStages * kAccCols);
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
  static_assert(kStages >= 2, "pipeline too shallow");
  static_assert(kTmemCols <= 512, "TMEM overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "bad BN");
};

template <bool GATEUP, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x, const GemmParams p) {
  using C = Cfg<GATEUP, BN>;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
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
  // A producer may spend up to its 1 s arrival limit waiting for rows from
  // other ranks; the other roles' waits allow for that.
  const uint64_t wait_ns = p.arrive ? 3000000000ull : 1000000000ull;
  const int total = __ldg(p.nb_off + p.E) * p.n_mblk;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      // Weights are streamed once when an expert has a single token block;
      // otherwise every token block's CTA reads the same weight tile, and it
      // must stay in L2 until they all have.
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      int arrived_e = -1;  // the expert whose rows are known to be here
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, mb, nb;
        decode_tile(tile, p, e, mb, nb);
        if (p.arrive && e != arrived_e) {
          rows_arrived(p.arrive + e, __ldg(p.counts + e), p.status, kFlagArrival);
          arrived_e = e;
        }
        const int wrow = e * p.w_rows + mb * kTileM;
        const int xrow = __ldg(p.offsets + e) + nb * BN;
        const int nblk = __ldg(p.nb_off + e + 1) - __ldg(p.nb_off + e);
        const uint64_t pol_w = nblk == 1 ? pol_stream : pol_keep;
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer, wait_ns)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          tma_load_2d(sa, &tm_w, &full[stage], kb * kTileK, wrow, pol_w);
          if (GATEUP)
            tma_load_2d(sa + C::kABytes, &tm_w, &full[stage], kb * kTileK, wrow + p.up_rows,
                        pol_w);
          tma_load_2d(sa + C::kNA * C::kABytes, &tm_x, &full[stage], kb * kTileK, xrow, pol_keep);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let every copy this thread issued land before the CTA can exit.
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t i = first; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), nullptr, nullptr, 0u,
                  100000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, mb, nb;
        decode_tile(tile, p, e, mb, nb);
        const int rows = min(BN, __ldg(p.counts + e) - nb * BN);
        const uint32_t n_mma = (uint32_t)((rows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(kTileM, n_mma);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, kFlagMma, wait_ns)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * C::kAccCols);
        const uint32_t d1 = d0 + BN;
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint64_t da0 = smem_desc_k_sw128(sa);
          const uint64_t da1 = smem_desc_k_sw128(sa + C::kABytes);
          const uint64_t db = smem_desc_k_sw128(sa + C::kNA * C::kABytes);
#pragma unroll
          for (int k4 = 0; k4 < kTileK / 16; ++k4) {
            const uint32_t accum = (kb | k4) != 0;
            umma_bf16(d0, da0 + 2u * k4, db + 2u * k4, idesc, accum);
            if (GATEUP) umma_bf16(d1, da1 + 2u * k4, db + 2u * k4, idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (C::kAccStages == 2) {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
        } else {
          acc_phase ^= 1u;
        }
      }
      // Every MMA this thread issued completes before TMEM is released.
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, mb, nb;
      decode_tile(tile, p, e, mb, nb);
      const int rows = min(BN, __ldg(p.counts + e) - nb * BN);
      const int n_mma = (rows + 15) & ~15;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, kFlagEpilogue, wait_ns)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::kAccCols);
      const int64_t row0 = __ldg(p.offsets + e) + nb * BN;
      const int64_t o0 = row0 * p.out_ld + mb * kTileM + r;
      for (int c0 = 0; c0 < n_mma; c0 += 16) {
        uint32_t g[16], u[16];
        tmem_ld16(tb + c0, g);
        if (GATEUP) tmem_ld16(tb + BN + c0, u);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = c0 + j;
          if (t < rows) {
            if (GATEUP) {
              const float v = silu_mul(__uint_as_float(g[j]), __uint_as_float(u[j]));
              static_cast<uint16_t*>(p.out)[o0 + (int64_t)t * p.out_ld] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(v));
            } else {
              static_cast<float*>(p.out)[o0 + (int64_t)t * p.out_ld] = __uint_as_float(g[j]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (C::kAccStages == 2) {
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        acc_phase ^= 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <bool GATEUP, int BN>
cudaError_t run(const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                cudaStream_t st) {
  using C = Cfg<GATEUP, BN>;
  static PerDevice configured;  // the shared-memory attribute, once per device
  int unused = 0;
  cudaError_t err = per_device(configured, &unused, [](int*) {
    return cudaFuncSetAttribute(grouped_gemm_kernel<GATEUP, BN>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  grouped_gemm_kernel<GATEUP, BN><<<device_sm_count(), kThreads, C::kSmemBytes, st>>>(tw, tx, p);
  return cudaGetLastError();
}

template <bool GATEUP>
cudaError_t dispatch_bn(int bn, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                        cudaStream_t st) {
  switch (bn) {
    case 16: return run<GATEUP, 16>(tw, tx, p, st);
    case 32: return run<GATEUP, 32>(tw, tx, p, st);
    case 64: return run<GATEUP, 64>(tw, tx, p, st);
    case 128: return run<GATEUP, 128>(tw, tx, p, st);
    case 256: return run<GATEUP, 256>(tw, tx, p, st);
    default: return cudaErrorInvalidValue;
  }
}

GemmParams base_params(const beam_moe_cfg& c, const Layout& L, char* ws) {
  GemmParams p;
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.nb_off = reinterpret_cast<const int32_t*>(ws + L.nb_off);
  p.E = c.n_experts;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);
  p.arrive = L.arrive ? reinterpret_cast<const int32_t*>(ws + L.arrive) : nullptr;
  p.next_tile = nullptr;  // static tile order here
  return p;
}

}  // namespace

cudaError_t launch_gateup(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13, char* ws,
                          cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx;
  cudaError_t err = encode_tmap_2d_bf16(&tw, w13, (uint64_t)H, (uint64_t)E * 2 * I, kTileK, kTileM);
  if (err != cudaSuccess) return err;
  err = encode_tmap_2d_bf16(&tx, ws + L.xp, (uint64_t)H, (uint64_t)L.A, kTileK, (uint32_t)L.bn);
  if (err != cudaSuccess) return err;
  GemmParams p = base_params(c, L, ws);
  p.out = ws + L.h;
  p.out_ld = I;
  p.nk = H / kTileK;
  p.w_rows = 2 * I;
  p.up_rows = I;
  p.n_mblk = I / kTileM;
  return dispatch_bn<true>(L.bn, tw, tx, p, st);
}

cudaError_t launch_gateup_light(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13,
                                char* ws, cudaStream_t st) {
  Layout M = L;
  M.bn = L.light_bn;
  M.nb_off = L.nbl_off;
  return launch_gateup(c, M, w13, ws, st);
}

cudaError_t launch_down_light(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2,
                              char* ws, cudaStream_t st) {
  Layout M = L;
  M.bn = L.light_bn;
  M.nb_off = L.nbl_off;
  return launch_down(c, M, w2, ws, st);
}

cudaError_t launch_down(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2, char* ws,
                        cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx;
  cudaError_t err = encode_tmap_2d_bf16(&tw, w2, (uint64_t)I, (uint64_t)E * H, kTileK, kTileM);
  if (err != cudaSuccess) return err;
  err = encode_tmap_2d_bf16(&tx, ws + L.h, (uint64_t)I, (uint64_t)L.A, kTileK, (uint32_t)L.bn);
  if (err != cudaSuccess) return err;
  GemmParams p = base_params(c, L, ws);
  p.out = ws + L.xp;  // fp32 y reuses the permuted-input rows
  p.out_ld = H;
  p.nk = I / kTileK;
  p.w_rows = H;
  p.up_rows = 0;
  p.arrive = nullptr;  // h rows are this rank's own
  p.n_mblk = H / kTileM;
  return dispatch_bn<false>(L.bn, tw, tx, p, st);
}

}  // namespace beam
