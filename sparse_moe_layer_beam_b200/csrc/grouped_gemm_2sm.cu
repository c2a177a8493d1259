// grouped_gemm_2sm.cu - the expert GEMMs for many rows per expert, on CTA
// pairs (tcgen05 cta_group::2). Same operations as grouped_gemm.cu:
//
//   gate/up:  [g | u] = W13_e x, h = silu(g) * u in FP32 -> bf16   (K = H)
//   down:     y = W2_e h -> fp32                                  (K = I)
//
// Under expert parallelism the down GEMM's epilogue stores each y row straight
// into the workspace of the rank the row came from (a peer store over NVLink
// between GPUs), so the return of y overlaps the tensor-core tiles instead of
// following them as a copy.
//
// One MMA covers 256 weight rows x up to 256 tokens. Each CTA of the pair
// holds 128 weight rows and half of the tokens in its shared memory and 128
// accumulator rows in its TMEM, so a CTA moves a third fewer operand bytes per
// FLOP than a single-CTA 128 x 256 tile, and the 128 x 256 FP32 accumulator
// (256 TMEM columns) is double-buffered: the epilogue of one tile overlaps the
// MMAs of the next.
//
// Gate/up rows are interleaved in 16-row blocks inside a CTA's 128 rows
// (gate 0-15, up 0-15, gate 16-31, ...), loaded with one 5-D TMA box, so that
// a warp's 32 TMEM lanes hold 16 gate rows and the 16 up rows of the same
// intermediate indices; lanes exchange halves with one shuffle.
//
// A CTA loads its half of a tile's token rows as one box of 64 rows when
// that covers them, else of 128: an expert with up to 128 rows then costs 64
// rows of operand reads per CTA and k-step, not 128. (Measured: one box per
// k-step beats an exact cover by several smaller boxes, and 8- to 32-row
// boxes run slower than the 64-row box although they move fewer bytes.)
//
// Tiles are handed out in order at run time: the even CTA's producer takes
// the next index from a counter in global memory and publishes it, through a
// small ring in both CTAs' shared memory, to every role of the pair. So the
// 74 pairs work on a window of consecutive tiles (those of one or two
// experts) however their speeds differ, instead of drifting apart over a
// static stride, which would spread the operands they share over more of L2.
//
// Roles (both CTAs have the same warps): warp 0 issues this CTA's TMA loads,
// whose completion is counted on the even CTA's barrier; warp 1 of the even
// CTA issues the pair's MMAs and commits to barriers in both CTAs; warps 2-5
// of each CTA drain their own TMEM and tell the even CTA's MMA thread. The
// pair allocates TMEM together and meets at a cluster barrier before freeing
// it. No load uses multicast. Every wait is bounded.
#include <cuda_bf16.h>
#include <string.h>

#include "grouped_gemm.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace beam {
namespace {

using gg::GemmParams;
using gg::decode_tile;
using gg::silu_mul;

constexpr int kThreads = 192;
constexpr int kTileSlots = 8;  // tile indices in flight between the fetching producer and the rest
// readers of each published index: the odd CTA's producer, the MMA thread and
// the four epilogue warps of each CTA
constexpr int kTileReaders = 1 + 1 + 2 * 4;
constexpr int kPairM = 256;  // weight rows per pair tile
constexpr int kPairN = 256;  // max tokens per pair tile (the token block)

// Tile -> (expert, weight block, token block). An expert's tiles run weight
// block by weight block, so that each weight tile is read from DRAM once while
// the expert's token rows stay in L2 - unless the token rows outweigh the
// weights (more rows than the expert has weight rows): then token block by
// token block, and the weights are what stays in L2.
__device__ __forceinline__ void decode_pair_tile(int tile, const GemmParams& p, int& e, int& mb,
                                                 int& nb) {
  decode_tile(tile, p, e, mb, nb);
  if (__ldg(p.counts + e) > p.w_rows) {
    const int nblk = __ldg(p.nb_off + e + 1) - __ldg(p.nb_off + e);
    const int local = mb * nblk + nb;
    nb = local / p.n_mblk;
    mb = local - nb * p.n_mblk;
  }
}

struct PairCfg {
  static constexpr int kABytes = 128 * kTileK * 2;  // this CTA's 128 weight rows
  static constexpr int kBBytes = 128 * kTileK * 2;  // room for this CTA's half of 256 tokens
  static constexpr int kRowBytes = kTileK * 2;      // one token row of a k-step
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 7;  // 225 KB of the 227 KB a CTA may use
  static constexpr int kAccCols = kPairN;  // FP32 accumulator columns per stage
  static constexpr int kTmemCols = 512;    // two accumulator stages
  static constexpr int kBarBytes = 512;  // mbarriers, TMEM address, abort flag, tile ring
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
  static_assert(kSmemBytes <= 232448, "dynamic shared memory above the sm_100 limit");
};

// EPRET: the down GEMM under expert parallelism, storing y rows to their
// source ranks (a separate instance, so that the plain epilogue stays lean).
template <bool GATEUP, bool EPRET>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                             const __grid_constant__ CUtensorMap tm_x,
                             const __grid_constant__ CUtensorMap tm_x64, const GemmParams p,
                             const __grid_constant__ EpReturn ret) {
  using C = PairCfg;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* tsfull = drain + 1;              // [kTileSlots] an index is in the ring
  uint64_t* tsempty = tsfull + kTileSlots;   // [kTileSlots] every reader has it (even CTA)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tsempty + kTileSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* ring = abort_flag + 1;       // [kTileSlots] tile index, -1: no more
  static_assert((2 * PairCfg::kStages + 5 + 2 * kTileSlots) * 8 + 8 + 4 * kTileSlots <=
                    PairCfg::kBarBytes,
                "barrier area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues MMAs
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's arrive.expect_tx + both CTAs' bytes
      mbar_init(&empty[s], 1);  // one multicast commit per consumed stage
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 128);  // epilogue threads of both CTAs
    }
    mbar_init(drain, 1);
    for (int s = 0; s < kTileSlots; ++s) {
      mbar_init(&tsfull[s], 1);
      mbar_init(&tsempty[s], kTileReaders);
    }
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
  // A producer may spend up to its 1 s arrival limit waiting for rows from
  // other ranks; the other roles' waits allow for that.
  const uint64_t wait_ns = p.arrive ? 3000000000ull : 1000000000ull;
  const int total = __ldg(p.nb_off + p.E) * p.n_mblk;
  // Next tile index of this pair, in order, for every role. The even CTA's
  // producer takes it from the counter and publishes it to both CTAs; the
  // others read it. -1: no tiles left; -2: a wait gave up (the role stops).
  int tslot = 0;
  uint32_t tphase = 0;
  // t: the counter value taken for this slot (taken one tile ahead, so that
  // the atomic's latency overlaps the previous tile's loads).
  auto publish_tile = [&](int t) -> int {
    // the readers' arrivals (some from the other CTA) come before the rewrite
    if (!mbar_wait(&tsempty[tslot], tphase ^ 1u, abort_flag, p.status, kFlagProducer, wait_ns,
                   true))
      return -2;
    const int tile = t < total ? t : -1;
    ring[tslot] = tile;
    st_cluster_u32(mapa_shared(smem_addr((const void*)&ring[tslot]), 1), (uint32_t)tile);
    mbar_arrive(&tsfull[tslot]);
    mbar_arrive_cluster(mapa_shared(smem_addr(&tsfull[tslot]), 1));
    if (++tslot == kTileSlots) {
      tslot = 0;
      tphase ^= 1u;
    }
    return tile;
  };
  // Without a counter (experts with about one token block each, where tiles
  // share no operands and the hand-out would only add latency), every role
  // walks this pair's static stride instead.
  const bool dynamic = p.next_tile != nullptr;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  int stile = pair;
  auto next_static = [&]() -> int {
    const int t = stile;
    stile += n_pairs;
    return t < total ? t : -1;
  };
  // whole_warp: all 32 lanes read (the epilogue warps; lane 0 then arrives
  // for the warp), else one thread reads and arrives.
  auto read_tile = [&](uint32_t flag, bool whole_warp) -> int {
    // the index may have been stored by the other CTA, released at cluster scope
    const bool got = mbar_wait(&tsfull[tslot], tphase, abort_flag, p.status, flag, wait_ns, true);
    // a warp leaves together, even if its lanes' waits ran out at different times
    if (whole_warp ? !__all_sync(0xffffffffu, got) : !got) return -2;
    const int tile = ring[tslot];
    if (whole_warp) __syncwarp();  // every lane has read the slot
    if (!whole_warp || lane == 0)
      mbar_arrive_cluster(mapa_shared(smem_addr(&tsempty[tslot]), 0));
    if (++tslot == kTileSlots) {
      tslot = 0;
      tphase ^= 1u;
    }
    return tile;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      int arrived_e = -1;  // the expert whose rows are known to be here
      int taken = (dynamic && leader) ? atomicAdd(p.next_tile, 1) : 0;
      for (;;) {
        const int tile = !dynamic ? next_static()
                         : leader ? publish_tile(taken)
                                  : read_tile(kFlagProducer, false);
        if (tile < 0) {
          ok = tile == -1;
          break;
        }
        if (dynamic && leader) taken = atomicAdd(p.next_tile, 1);  // used at the next tile
        int e, mb, nb;
        decode_pair_tile(tile, p, e, mb, nb);
        if (p.arrive && e != arrived_e) {
          rows_arrived(p.arrive + e, __ldg(p.counts + e), p.status, kFlagArrival);
          arrived_e = e;
        }
        const int rows = min(kPairN, __ldg(p.counts + e) - nb * kPairN);
        const int half = ((rows + 15) & ~15) >> 1;  // 8 .. 128
        const int xrow = __ldg(p.offsets + e) + nb * kPairN + (int)rank * half;
        const bool box64 = half <= 64;
        const CUtensorMap* tmx = box64 ? &tm_x64 : &tm_x;
        const uint32_t stage_tx = 2u * (uint32_t)(C::kABytes + (box64 ? 64 : 128) * C::kRowBytes);
        const int nblk = __ldg(p.nb_off + e + 1) - __ldg(p.nb_off + e);
        const uint64_t pol_w = nblk == 1 ? pol_stream : pol_keep;
        // first weight row of this CTA's 128 (down) or first intermediate
        // index of its 64 gate/up pairs
        const int w0 = GATEUP ? mb * 128 + (int)rank * 64
                              : e * p.w_rows + mb * kPairM + (int)rank * 128;
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer, wait_ns)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
          const uint32_t bar = mapa_shared(smem_addr(&full[stage]), 0);
          const int kx = kb * kTileK;
          if (GATEUP) {
            tma_load_5d_pair(sa, &tm_w, bar, kx, 0, 0, w0 / 16, e, pol_w);
          } else {
            tma_load_2d_pair(sa, &tm_w, bar, kx, w0, pol_w);
          }
          tma_load_2d_pair(sa + C::kABytes, tmx, bar, kx, xrow, pol_keep);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // The even CTA's full barriers count both CTAs' copies: wait for the
      // last ones to land before either CTA can leave.
      if (leader) {
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
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (;;) {
        const int tile = dynamic ? read_tile(kFlagMma, false) : next_static();
        if (tile < 0) break;
        int e, mb, nb;
        decode_pair_tile(tile, p, e, mb, nb);
        const int rows = min(kPairN, __ldg(p.counts + e) - nb * kPairN);
        const uint32_t n_mma = (uint32_t)((rows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(kPairM, n_mma);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, kFlagMma, wait_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * C::kAccCols);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint64_t da = smem_desc_k_sw128(sa);
          const uint64_t db = smem_desc_k_sw128(sa + C::kABytes);
#pragma unroll
          for (int k4 = 0; k4 < kTileK / 16; ++k4)
            umma_bf16_pair(d, da + 2u * k4, db + 2u * k4, idesc, (kb | k4) != 0);
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every MMA of the pair completes before TMEM is released.
      umma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    int acc = 0;
    uint32_t acc_phase = 0;
    for (;;) {
      const int tile = dynamic ? read_tile(kFlagEpilogue, true) : next_static();
      if (tile < 0) break;
      int e, mb, nb;
      decode_pair_tile(tile, p, e, mb, nb);
      const int rows = min(kPairN, __ldg(p.counts + e) - nb * kPairN);
      const int n_mma = (rows + 15) & ~15;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, kFlagEpilogue, wait_ns)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::kAccCols);
      const int64_t row0 = __ldg(p.offsets + e) + nb * kPairN;
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
      } else if (!EPRET) {
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
      } else {
        // each row to its source rank's returned-y row of the same slot
        const int col = mb * kPairM + (int)rank * 128 + q * 32 + lane;
        for (int c0 = 0; c0 < n_mma; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < rows) {
              const uint32_t code = (uint32_t)__ldg(ret.src + row0 + c0 + j);
              const int s = (int)(code >> kEpSlotBits);
              const int64_t slot = code & ((1u << kEpSlotBits) - 1u);
              if (s < ret.world && slot < ret.slots) {
                reinterpret_cast<float*>(ret.peer[s] + ret.yret_off)[slot * p.out_ld + col] =
                    __uint_as_float(v[j]);
              } else if (lane == 0) {  // never stored through
                atomicOr(p.status, kFlagBadReturn);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(mapa_shared(smem_addr(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (EPRET) __threadfence_system();  // the sources combine these rows on other GPUs
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // both CTAs done with TMEM and with each other's memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

template <bool GATEUP, bool EPRET>
cudaError_t run_pair(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& tx64,
                     const GemmParams& p, const EpReturn& ret, cudaStream_t st) {
  // Per device: the shared-memory attribute and the number of CTA pairs that
  // can be resident at once (a pair needs two SMs of one GPC). The grid is
  // exactly that many pairs, so no pair waits for another to finish.
  static PerDevice pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PairCfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int resident_pairs = 0;
  cudaError_t err = per_device(pairs, &resident_pairs, [&cfg](int* v) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<GATEUP, EPRET>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t probe = cfg;
    probe.gridDim = dim3((unsigned)(device_sm_count() & ~1));
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<GATEUP, EPRET>, &probe);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    *v = clusters < device_sm_count() / 2 ? clusters : device_sm_count() / 2;
    return cudaSuccess;
  });
  if (err != cudaSuccess) return err;
  if (p.next_tile) {
    err = cudaMemsetAsync(p.next_tile, 0, sizeof(int), st);
    if (err != cudaSuccess) return err;
  }
  cfg.gridDim = dim3((unsigned)(2 * resident_pairs));
  return cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<GATEUP, EPRET>, tw, tx, tx64, p, ret);
}

// Token-row boxes of 128 and 64 rows over the same matrix.
cudaError_t encode_xmaps(CUtensorMap* m128, CUtensorMap* m64, const void* base, uint64_t cols,
                         uint64_t rows) {
  cudaError_t err = encode_tmap_2d_bf16(m128, base, cols, rows, kTileK, 128);
  if (err != cudaSuccess) return err;
  return encode_tmap_2d_bf16(m64, base, cols, rows, kTileK, 64);
}

GemmParams base_params(const beam_moe_cfg& c, const Layout& L, char* ws) {
  GemmParams p;
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.nb_off = reinterpret_cast<const int32_t*>(ws + L.nb_off);
  p.E = c.n_experts;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);
  p.arrive = L.arrive ? reinterpret_cast<const int32_t*>(ws + L.arrive) : nullptr;
  // Tiles handed out at run time once experts average more than one 256-token
  // block (then an expert's tiles share operands through L2); the counter is
  // a word of the status area past the status word itself.
  const bool dynamic = (double)L.A > (double)kPairN * c.n_experts;
  p.next_tile = dynamic ? reinterpret_cast<int*>(ws + L.status) + kTileCounterWord : nullptr;
  return p;
}

}  // namespace

bool pair_gemm_supported(const beam_moe_cfg& c) {
  return c.hidden % kPairM == 0 && c.inter % 128 == 0;
}

cudaError_t launch_gateup_pair(const beam_moe_cfg& c, const Layout& L, const uint16_t* w13,
                               char* ws, cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx, tx64;
  cudaError_t err = encode_tmap_w13_interleaved(&tw, w13, (uint64_t)H, (uint64_t)I, (uint64_t)E);
  if (err != cudaSuccess) return err;
  err = encode_xmaps(&tx, &tx64, ws + L.xp, (uint64_t)H, (uint64_t)L.A);
  if (err != cudaSuccess) return err;
  GemmParams p = base_params(c, L, ws);
  p.out = ws + L.h;
  p.out_ld = I;
  p.nk = H / kTileK;
  p.w_rows = 2 * I;
  p.up_rows = I;
  p.n_mblk = I / 128;  // 128 intermediate indices (gate + up) per pair tile
  EpReturn none;
  memset(&none, 0, sizeof(none));
  return run_pair<true, false>(tw, tx, tx64, p, none, st);
}

cudaError_t launch_down_pair(const beam_moe_cfg& c, const Layout& L, const uint16_t* w2,
                             char* ws, cudaStream_t st, const EpReturn* ret) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  CUtensorMap tw, tx, tx64;
  cudaError_t err = encode_tmap_2d_bf16(&tw, w2, (uint64_t)I, (uint64_t)E * H, kTileK, 128);
  if (err != cudaSuccess) return err;
  err = encode_xmaps(&tx, &tx64, ws + L.h, (uint64_t)I, (uint64_t)L.A);
  if (err != cudaSuccess) return err;
  GemmParams p = base_params(c, L, ws);
  p.out = ws + L.xp;  // fp32 y reuses the permuted-input rows
  p.out_ld = H;
  p.nk = I / kTileK;
  p.w_rows = H;
  p.up_rows = 0;
  p.arrive = nullptr;  // h rows are this rank's own
  p.n_mblk = H / kPairM;
  if (ret && ret->src) return run_pair<false, true>(tw, tx, tx64, p, *ret, st);
  EpReturn none;
  memset(&none, 0, sizeof(none));
  return run_pair<false, false>(tw, tx, tx64, p, none, st);
}

}  // namespace beam
