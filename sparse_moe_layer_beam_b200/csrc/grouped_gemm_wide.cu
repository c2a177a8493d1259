// grouped_gemm_wide.cu - the expert GEMMs for experts with hundreds of rows or
// more, on CTA pairs with 512-token tiles. Same operations as
// grouped_gemm.cu and grouped_gemm_2sm.cu ("Welcome Beam", section "Mixture
// of Experts": SwiGLU experts; section "Residual Stream": the SwiGLU product
// in FP32):
//
//   gate/up:  [g | u] = W13_e x, h = silu(g) * u in FP32 -> bf16   (K = H)
//   down:     y = W2_e h -> fp32                                  (K = I)
//
// At many rows per expert the CTA-pair kernel with 256-token tiles is bounded
// by operand feed from L2: per k-step of 64 a CTA reads 128 weight rows and
// 128 token rows (32 KB) for 4.2 MFLOP, 64 bytes per clock at the full MMA
// rate. Here one pair tile covers 256 weight rows x 512 tokens as two MMA
// accumulators that share the weight tile: a CTA reads 16 KB of weights and
// two 16 KB token halves per k-step for twice the FLOPs, 47 bytes per clock.
//
// The two 128 x 256 FP32 accumulators fill the CTA's 512 TMEM columns, so
// they are not double-buffered. Two groups of four epilogue warps drain them
// at once, each accumulator as soon as its last MMA completes, and the MMA
// thread starts the next tile on accumulator 0 as soon as it is drained,
// issuing accumulator 1's MMAs for the stages it has passed once that one is
// drained too (a stage is released only after both accumulators have read
// it). A tile with at most 256 rows uses accumulator 0 alone.
//
// Roles: warp 0 issues this CTA's TMA loads (completion counted on the even
// CTA's barrier), warp 1 of the even CTA issues the pair's MMAs, warps 2-5
// drain accumulator 0 and warps 6-9 accumulator 1 of their own CTA. No load
// uses multicast. Every wait is bounded.
#include <cuda_bf16.h>
#include <string.h>

#include "grouped_gemm.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace beam {
namespace {

using gg::GemmParams;
using gg::silu_mul;

constexpr int kThreads = 320;
constexpr int kPairM = 256;   // weight rows per pair tile
constexpr int kSubN = 256;    // tokens per accumulator (one MMA's N)
constexpr int kWideN = 512;   // tokens per pair tile

struct WideCfg {
  static constexpr int kABytes = 128 * kTileK * 2;  // this CTA's 128 weight rows
  static constexpr int kBBytes = 128 * kTileK * 2;  // room for this CTA's half of 256 tokens
  static constexpr int kRowBytes = kTileK * 2;      // one token row of a k-step
  static constexpr int kStageBytes = kABytes + 2 * kBBytes;
  static constexpr int kStages = 4;
  static constexpr int kTmemCols = 512;  // accumulator 0: columns 0-255, 1: 256-511
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
  static_assert(kSmemBytes <= 232448, "dynamic shared memory above the sm_100 limit");
};

// mbarrier phase test that never suspends the thread (the MMA issuer polls
// accumulator 1 between its MMAs).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Tile -> (expert, weight block, 512-token block), with p.nb_off the prefix
// of 512-row blocks per expert. An expert's tiles run weight block by weight
// block, so each weight tile is read from DRAM once while the expert's token
// rows stay in L2, unless its token rows outweigh its weights (more rows than
// weight rows): then token block by token block.
__device__ __forceinline__ void decode_wide_tile(int tile, const GemmParams& p, int& e, int& mb,
                                                 int& nb) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.nb_off + mid) * p.n_mblk <= tile) lo = mid;
    else hi = mid - 1;
  }
  e = lo;
  const int base = __ldg(p.nb_off + e);
  const int nblk = __ldg(p.nb_off + e + 1) - base;
  const int local = tile - base * p.n_mblk;
  if (__ldg(p.counts + e) > p.w_rows) {
    nb = local / p.n_mblk;
    mb = local - nb * p.n_mblk;
  } else {
    mb = local / nblk;
    nb = local - mb * nblk;
  }
}

// Rows of the tile's two 256-token sub-blocks.
__device__ __forceinline__ void sub_rows(const GemmParams& p, int e, int nb, int& r0, int& r1) {
  const int rows = min(kWideN, __ldg(p.counts + e) - nb * kWideN);
  r0 = min(kSubN, rows);
  r1 = rows - r0;
}

template <bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_wide_kernel(const __grid_constant__ CUtensorMap tm_w,
                             const __grid_constant__ CUtensorMap tm_x,
                             const __grid_constant__ CUtensorMap tm_x64, const GemmParams p) {
  using C = WideCfg;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2] accumulator i holds a finished tile
  uint64_t* tempty = tfull + 2;      // [2] accumulator i has been drained by both CTAs
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues MMAs
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 128);  // one epilogue group of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_x64);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int total = __ldg(p.nb_off + p.E) * p.n_mblk;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int e, mb, nb, r0, r1;
        decode_wide_tile(tile, p, e, mb, nb);
        sub_rows(p, e, nb, r0, r1);
        const int half0 = ((r0 + 15) & ~15) >> 1;  // 8 .. 128
        const int half1 = ((r1 + 15) & ~15) >> 1;  // 0 .. 128
        const int base = __ldg(p.offsets + e) + nb * kWideN;
        const int x0 = base + (int)rank * half0;
        const int x1 = base + kSubN + (int)rank * half1;
        const bool b0_64 = half0 <= 64, b1_64 = half1 <= 64;
        const uint32_t stage_tx =
            2u * (uint32_t)(C::kABytes + (b0_64 ? 64 : 128) * C::kRowBytes +
                            (half1 ? (b1_64 ? 64 : 128) * C::kRowBytes : 0));
        const int nblk = __ldg(p.nb_off + e + 1) - __ldg(p.nb_off + e);
        const uint64_t pol_w = nblk == 1 ? pol_stream : pol_keep;
        const int w0 = GATEUP ? mb * 128 + (int)rank * 64
                              : e * p.w_rows + mb * kPairM + (int)rank * 128;
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
          const uint32_t bar = mapa_shared(smem_addr(&full[stage]), 0);
          const int kx = kb * kTileK;
          if (GATEUP) tma_load_5d_pair(sa, &tm_w, bar, kx, 0, 0, w0 / 16, e, pol_w);
          else tma_load_2d_pair(sa, &tm_w, bar, kx, w0, pol_w);
          tma_load_2d_pair(sa + C::kABytes, b0_64 ? &tm_x64 : &tm_x, bar, kx, x0, pol_keep);
          if (half1)
            tma_load_2d_pair(sa + C::kABytes + C::kBBytes, b1_64 ? &tm_x64 : &tm_x, bar, kx, x1,
                             pol_keep);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {  // both CTAs' last copies land before either can leave
        const int64_t first = issued > STAGES ? issued - STAGES : 0;
        for (int64_t i = first; i < issued; ++i)
          mbar_wait(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), nullptr, nullptr, 0u,
                    100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // --------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t uses0 = 0, uses1 = 0;  // tiles each accumulator has taken so far
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int e, mb, nb, r0, r1;
        decode_wide_tile(tile, p, e, mb, nb);
        sub_rows(p, e, nb, r0, r1);
        const uint32_t n0 = (uint32_t)((r0 + 15) & ~15), n1 = (uint32_t)((r1 + 15) & ~15);
        const uint32_t idesc0 = idesc_bf16_f32(kPairM, n0);
        const uint32_t idesc1 = n1 ? idesc_bf16_f32(kPairM, n1) : 0u;
        const bool need1 = n1 != 0;
        // accumulator 0 must be drained before this tile's first MMA
        if (!mbar_wait(&tempty[0], (uses0 & 1u) ^ 1u, abort_flag, p.status, kFlagMma)) break;
        tc_fence_after();
        bool free1 = !need1;
        int pend = 0;     // first k-step whose accumulator-1 MMAs are still to issue
        int pstage = stage;  // its stage
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint64_t da = smem_desc_k_sw128(sa);
          const uint64_t db0 = smem_desc_k_sw128(sa + C::kABytes);
#pragma unroll
          for (int k4 = 0; k4 < kTileK / 16; ++k4)
            umma_bf16_pair(tmem_base, da + 2u * k4, db0 + 2u * k4, idesc0, (kb | k4) != 0);
          if (need1) {
            if (!free1) {
              // poll; block once every stage of the ring waits on accumulator 1
              free1 = mbar_test_wait(&tempty[1], (uses1 & 1u) ^ 1u);
              if (!free1 && kb - pend + 1 >= STAGES) {
                if (!mbar_wait(&tempty[1], (uses1 & 1u) ^ 1u, abort_flag, p.status, kFlagMma)) {
                  ok = false;
                  break;
                }
                free1 = true;
              }
              if (free1) tc_fence_after();
            }
            if (free1) {
              for (; pend <= kb; ++pend) {
                const uint32_t pa = smem_addr(smem + pstage * C::kStageBytes);
                const uint64_t pda = smem_desc_k_sw128(pa);
                const uint64_t pdb1 = smem_desc_k_sw128(pa + C::kABytes + C::kBBytes);
#pragma unroll
                for (int k4 = 0; k4 < kTileK / 16; ++k4)
                  umma_bf16_pair(tmem_base + kSubN, pda + 2u * k4, pdb1 + 2u * k4, idesc1,
                                 (pend | k4) != 0);
                umma_commit_pair(&empty[pstage], 0x3);
                if (++pstage == STAGES) pstage = 0;
              }
            }
          } else {
            umma_commit_pair(&empty[stage], 0x3);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[0], 0x3);  // accumulator 0 is complete
        ++uses0;
        if (need1) {
          if (!free1) {
            if (!mbar_wait(&tempty[1], (uses1 & 1u) ^ 1u, abort_flag, p.status, kFlagMma)) break;
            tc_fence_after();
          }
          for (; pend < p.nk; ++pend) {
            const uint32_t pa = smem_addr(smem + pstage * C::kStageBytes);
            const uint64_t pda = smem_desc_k_sw128(pa);
            const uint64_t pdb1 = smem_desc_k_sw128(pa + C::kABytes + C::kBBytes);
#pragma unroll
            for (int k4 = 0; k4 < kTileK / 16; ++k4)
              umma_bf16_pair(tmem_base + kSubN, pda + 2u * k4, pdb1 + 2u * k4, idesc1,
                             (pend | k4) != 0);
            umma_commit_pair(&empty[pstage], 0x3);
            if (++pstage == STAGES) pstage = 0;
          }
          umma_commit_pair(&tfull[1], 0x3);
          ++uses1;
        }
      }
      // Every MMA of the pair completes before TMEM is released.
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int grp = (warp - 2) >> 2;  // the accumulator this warp drains
    const int q = warp & 3;           // TMEM lane quadrant of this warp
    uint32_t uses = 0;
    for (int tile = pair; tile < total; tile += n_pairs) {
      int e, mb, nb, r0, r1;
      decode_wide_tile(tile, p, e, mb, nb);
      sub_rows(p, e, nb, r0, r1);
      const int rows = grp == 0 ? r0 : r1;
      if (rows == 0) continue;  // accumulator 1 unused by this tile
      const int n_mma = (rows + 15) & ~15;
      if (!mbar_wait(&tfull[grp], uses & 1u, abort_flag, p.status, kFlagEpilogue)) break;
      ++uses;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kSubN);
      const int64_t row0 = __ldg(p.offsets + e) + nb * kWideN + grp * kSubN;
      if (GATEUP) {
        // lanes 0-15: gate rows, 16-31: up rows of 16 intermediate indices
        const int idx = mb * 128 + (int)rank * 64 + q * 16 + (lane & 15);
        const int tsel = (lane >> 4) * 8;  // this lane's half of each 16 tokens
        uint16_t* out = static_cast<uint16_t*>(p.out) + idx;
        for (int c0 = 0; c0 < n_mma; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t send = lane < 16 ? v[8 + j] : v[j];
            const float other = __uint_as_float(__shfl_xor_sync(0xffffffffu, send, 16));
            const float g = lane < 16 ? __uint_as_float(v[j]) : other;
            const float u = lane < 16 ? other : __uint_as_float(v[8 + j]);
            const int t = c0 + tsel + j;
            if (t < rows)
              out[(row0 + t) * p.out_ld] = __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(g, u)));
          }
        }
      } else {
        const int col = mb * kPairM + (int)rank * 128 + q * 32 + lane;
        float* out = static_cast<float*>(p.out) + col;
        for (int c0 = 0; c0 < n_mma; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < rows) out[(row0 + c0 + j) * p.out_ld] = __uint_as_float(v[j]);
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_addr(&tempty[grp]), 0));
    }
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // both CTAs done with TMEM and with each other's memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

template <bool GATEUP>
cudaError_t run_wide(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& tx64,
                     const GemmParams& p, cudaStream_t st) {
  static PerDevice pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = WideCfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int resident_pairs = 0;
  cudaError_t err = per_device(pairs, &resident_pairs, [&cfg](int* v) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<GATEUP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         WideCfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t probe = cfg;
    probe.gridDim = dim3((unsigned)(device_sm_count() & ~1));
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_wide_kernel<GATEUP>, &probe);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    *v = clusters < device_sm_count() / 2 ? clusters : device_sm_count() / 2;
    return cudaSuccess;
  });
  if (err != cudaSuccess) return err;
  cfg.gridDim = dim3((unsigned)(2 * resident_pairs));
  return cudaLaunchKernelEx(&cfg, grouped_gemm_wide_kernel<GATEUP>, tw, tx, tx64, p);
}

cudaError_t encode_xmaps(CUtensorMap* m128, CUtensorMap* m64, const void* base, uint64_t cols,
                         uint64_t rows) {
  cudaError_t err = encode_tmap_2d_bf16(m128, base, cols, rows, kTileK, 128);
  if (err != cudaSuccess) return err;
  return encode_tmap_2d_bf16(m64, base, cols, rows, kTileK, 64);
}

GemmParams wide_params(const beam_moe_cfg& c, const Layout& L, char* ws) {
  GemmParams p;
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.nb_off = reinterpret_cast<const int32_t*>(ws + L.nb2_off);  // 512-row blocks (bn = 256)
  p.E = c.n_experts;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);
  return p;
}

}  // namespace

cudaError_t launch_gateup_wide(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13,
                               char* ws, cudaStream_t st) {
  if (L.bn != 256) return cudaErrorInvalidValue;  // nb2_off must count 512-row blocks
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx, tx64;
  cudaError_t err = encode_tmap_w13_interleaved(&tw, w13, (uint64_t)H, (uint64_t)I, (uint64_t)E);
  if (err != cudaSuccess) return err;
  err = encode_xmaps(&tx, &tx64, ws + L.xp, (uint64_t)H, (uint64_t)L.A);
  if (err != cudaSuccess) return err;
  GemmParams p = wide_params(c, L, ws);
  p.out = ws + L.h;
  p.out_ld = I;
  p.nk = H / kTileK;
  p.w_rows = 2 * I;
  p.up_rows = I;
  p.n_mblk = I / 128;  // 128 intermediate indices (gate + up) per pair tile
  return run_wide<true>(tw, tx, tx64, p, st);
}

cudaError_t launch_down_wide(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2, char* ws,
                             cudaStream_t st) {
  if (L.bn != 256) return cudaErrorInvalidValue;
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx, tx64;
  cudaError_t err = encode_tmap_2d_bf16(&tw, w2, (uint64_t)I, (uint64_t)E * H, kTileK, 128);
  if (err != cudaSuccess) return err;
  err = encode_xmaps(&tx, &tx64, ws + L.h, (uint64_t)I, (uint64_t)L.A);
  if (err != cudaSuccess) return err;
  GemmParams p = wide_params(c, L, ws);
  p.out = ws + L.xp;  // fp32 y reuses the permuted-input rows
  p.out_ld = H;
  p.nk = I / kTileK;
  p.w_rows = H;
  p.up_rows = 0;
  p.n_mblk = H / kPairM;
  return run_wide<false>(tw, tx, tx64, p, st);
}

}  // namespace beam
