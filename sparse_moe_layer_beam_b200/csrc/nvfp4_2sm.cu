// nvfp4_2sm.cu - the NVFP4 down GEMM of the Beam MoE block (y = W2 h, FP4
// codes with E4M3 block scales, FP32 accumulation) on CTA pairs, for many
// rows per expert. Same operation as the down kernel of nvfp4.cu.
//
// One tcgen05.mma.cta_group::2 covers 256 weight rows x up to 256 tokens.
// Each CTA of the pair holds 128 weight rows and half of the tokens in its
// shared memory, so per FLOP it moves half the operand bytes of the
// single-CTA 128 x 128 tile; its TMEM holds its 128 accumulator rows.
//
// Block scales: the MMA reads, in each CTA's own TMEM, the scales of that
// CTA's 128 A rows (lane m, column base + m/32) and of all N token rows
// (column base + n/32, lanes replicated over the four lane quarters). So
// each CTA loads its own A scale atoms and the atoms of both 128-row token
// blocks, and copies them with its own tcgen05.cp.
//
// Roles (both CTAs have the same warps): warp 0 issues this CTA's TMA loads
// (codes complete on the even CTA's barrier, scale atoms on this CTA's);
// warp 1 of the even CTA issues the pair's MMAs and commits to barriers in
// both CTAs; warps 2-3 copy this CTA's scales to TMEM and tell the even
// CTA's MMA thread; warps 4-11 drain this CTA's accumulator into registers,
// hand it back, and store y. No load uses multicast. Every wait is bounded.
#include "internal.h"
#include "sm100.cuh"
#include "sm100_fp4.cuh"

namespace beam {
namespace {

constexpr int kPM = 256;              // weight rows per pair tile
constexpr int kPN = 256;              // max tokens per pair tile
constexpr int kCode = 128 * 128;      // bytes: 128 rows x 256 FP4 elements of K
constexpr int kAtoms = 4 * 512;       // scale atoms of 128 rows x 256 elements of K
constexpr int kEpiWarps = 8;
constexpr int kFirstEpi = 4;
constexpr int kThreads = 32 * (kFirstEpi + kEpiWarps);

struct Pair4Params {
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* nb_off;   // prefix of 128-row token blocks per expert
  const int32_t* nb2_off;  // prefix of 256-row token tiles per expert
  const uint8_t* w_sf;     // W2 scales, atom layout over the stacked rows
  const uint8_t* x_sf;     // h scales, atom layout over the padded rows
  float* y;                // fp32 [A][H]
  int E, H;
  int nk;                  // K / 256
  int sf_chunks;           // K / 64
  float acc_scale;
  unsigned* status;
};

struct P4Cfg {
  static constexpr int kStageBytes = 2 * kCode + 3 * kAtoms;  // A, B codes; A, B0, B1 atoms
  static constexpr int kStages = (220 * 1024) / kStageBytes;
  static constexpr int kAccCols = kPN;
  static constexpr int kSfCols = 16 + 32;  // A: 4 per chunk; B: 8 per chunk
  static constexpr int kSfBufs = 4;
  static constexpr int kTmemCols = 512;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256;
  static_assert(kAccCols + kSfBufs * kSfCols <= kTmemCols, "TMEM overflow");
  static_assert(kStages >= 3, "pipeline too shallow");
  static_assert((4 * kStages + 5) * 8 + 8 <= 256, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void decode_ptile(int tile, const Pair4Params& p, int n_mblk, int& e,
                                             int& mb, int& tt) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.nb2_off + mid) * n_mblk <= tile) lo = mid;
    else hi = mid - 1;
  }
  e = lo;
  const int base = __ldg(p.nb2_off + e);
  const int ntt = __ldg(p.nb2_off + e + 1) - base;
  const int local = tile - base * n_mblk;
  mb = local / ntt;
  tt = local - mb * ntt;
}

__global__ void __launch_bounds__(kThreads, 1)
    down_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tm_w,
                           const __grid_constant__ CUtensorMap tm_x, const Pair4Params p) {
  using C = P4Cfg;
  constexpr int STAGES = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // stage: [A codes][B codes][A atoms][B block 0 atoms][B block 1 atoms]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);  // even CTA
  uint64_t* sffull = full + STAGES;     // this CTA's scale atoms landed
  uint64_t* sfready = sffull + STAGES;  // even CTA: both CTAs' scales are in TMEM
  uint64_t* empty = sfready + STAGES;   // the pair's MMAs of the stage are done
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;         // even CTA
  uint64_t* drain = tempty + 1;         // [0] MMA issuer, [1], [2] scale copiers
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues MMAs
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int n_mblk = p.H / kPM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sffull[s], 1);
      mbar_init(&sfready[s], 4);  // two copier warps in each CTA
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * 32 * kEpiWarps);
    for (int d = 0; d < 3; ++d) mbar_init(&drain[d], 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t tsf = tmem_base + (uint32_t)C::kAccCols;
  const int total = __ldg(p.nb2_off + p.E) * n_mblk;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint64_t pol_keep = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int e, mb, tt;
        decode_ptile(tile, p, n_mblk, e, mb, tt);
        const int rows = min(kPN, __ldg(p.counts + e) - tt * kPN);
        const int half = ((rows + 15) & ~15) >> 1;
        const int blk0 = __ldg(p.nb_off + e) + 2 * tt;  // first 128-row token block
        const int nbb = (rows + 127) >> 7;
        const int xrow = blk0 * 128 + (int)rank * half;
        const int wrow = e * p.H + mb * kPM + (int)rank * 128;
        const uint32_t sf_bytes = (uint32_t)((1 + nbb) * kAtoms);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* ssf = sa + 2 * kCode;
          if (leader) mbar_arrive_expect_tx(&full[stage], 4 * kCode);
          const uint32_t bar = mapa_shared(smem_addr(&full[stage]), 0);
          const int kx = kb * 128;  // byte coordinate along K
          tma_load_2d_pair(sa, &tm_w, bar, kx, wrow, pol_keep);
          tma_load_2d_pair(sa + kCode, &tm_x, bar, kx, xrow, pol_keep);
          mbar_arrive_expect_tx(&sffull[stage], sf_bytes);
          bulk_load(ssf, p.w_sf + ((size_t)(wrow / 128) * p.sf_chunks + kb * 4) * 512, kAtoms,
                    &sffull[stage], pol_keep);
          for (int b = 0; b < nbb; ++b)
            bulk_load(ssf + (1 + b) * kAtoms,
                      p.x_sf + ((size_t)(blk0 + b) * p.sf_chunks + kb * 4) * 512, kAtoms,
                      &sffull[stage], pol_keep);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Let this CTA's copies land before it can leave: the scale atoms on
      // its own barriers, the codes of both CTAs on the even CTA's.
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t i = first; i < issued; ++i) {
        mbar_wait(&sffull[i % STAGES], (uint32_t)((i / STAGES) & 1), nullptr, nullptr, 0u,
                  100000000ull);
        if (leader)
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
      uint32_t acc_phase = 0;
      int sfbuf = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int e, mb, tt;
        decode_ptile(tile, p, n_mblk, e, mb, tt);
        const int rows = min(kPN, __ldg(p.counts + e) - tt * kPN);
        const uint32_t n_mma = (uint32_t)((rows + 15) & ~15);
        const uint32_t idesc = idesc_nvf4(kPM, n_mma);
        if (!mbar_wait(tempty, acc_phase ^ 1u, abort_flag, p.status, kFlagMma)) break;
        tc_fence_after();
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma) ||
              !mbar_wait(&sfready[stage], phase, abort_flag, p.status, kFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint32_t tsa = tsf + (uint32_t)(sfbuf * C::kSfCols);
          const uint32_t tsb = tsa + 16;
          if (++sfbuf == C::kSfBufs) sfbuf = 0;
          const uint64_t da = smem_desc_k_sw128(sa);
          const uint64_t db = smem_desc_k_sw128(sa + kCode);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_nvf4_pair(tmem_base, da + 2u * j, db + 2u * j, idesc, tsa + 4 * j, tsb + 8 * j,
                           (kb | j) != 0);
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull, 0x3);
        acc_phase ^= 1u;
      }
      // Every MMA of the pair completes before TMEM is released.
      umma_commit_pair(&drain[0], 0x1);
      mbar_wait(&drain[0], 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else if (warp < kFirstEpi) {
    if (lane == 0) {
      // ------------------------------------------------------ scale copiers
      // Warp 2 copies chunks 0-1 of the stage's atoms, warp 3 chunks 2-3:
      // chunk j of the A atoms to columns 4j of the scale buffer, chunk j of
      // token block b to 16 + 8j + 4b. Stage i uses buffer i mod kSfBufs,
      // which the MMAs of stage i - kSfBufs read: they must be done.
      const int j0 = 2 * (warp - 2);
      int64_t i = 0;
      int stage = 0;
      uint32_t phase = 0;
      int sfbuf = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += n_pairs) {
        int e, mb, tt;
        decode_ptile(tile, p, n_mblk, e, mb, tt);
        (void)mb;
        const int rows = min(kPN, __ldg(p.counts + e) - tt * kPN);
        const int nbb = (rows + 127) >> 7;
        for (int kb = 0; kb < p.nk; ++kb, ++i) {
          if (!mbar_wait(&sffull[stage], phase, abort_flag, p.status, kFlagMma)) {
            ok = false;
            break;
          }
          if (i >= C::kSfBufs) {
            const int64_t k = i - C::kSfBufs;
            if (!mbar_wait(&empty[k % STAGES], (uint32_t)((k / STAGES) & 1), abort_flag,
                           p.status, kFlagMma)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          const uint32_t ssf = smem_addr(smem + stage * C::kStageBytes) + 2 * kCode;
          const uint32_t tsa = tsf + (uint32_t)(sfbuf * C::kSfCols);
          const uint32_t tsb = tsa + 16;
          if (++sfbuf == C::kSfBufs) sfbuf = 0;
#pragma unroll
          for (int j = j0; j < j0 + 2; ++j) {
            tmem_cp_sf_atom(tsa + 4 * j, smem_desc_sf_atom(ssf + 512 * j));
            for (int b = 0; b < nbb; ++b)
              tmem_cp_sf_atom(tsb + 8 * j + 4 * b,
                              smem_desc_sf_atom(ssf + (1 + b) * kAtoms + 512 * j));
          }
          tc_commit_to(&sfready[stage], 0x1);  // the even CTA's barrier
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      uint64_t* own = &drain[1 + (warp - 2)];
      umma_commit(own);  // this warp's copies are done before TMEM is freed
      mbar_wait(own, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    // lane quarter q holds weight rows (H indices) mb*256 + rank*128 + 32q
    // + lane; this warp takes token columns [c_beg, c_beg + 128)
    const int q = warp & 3;
    const int c_beg = ((warp - kFirstEpi) >> 2) * 128;
    uint32_t acc_phase = 0;
    const uint32_t tempty_leader = mapa_shared(smem_addr(tempty), 0);
    for (int tile = pair; tile < total; tile += n_pairs) {
      int e, mb, tt;
      decode_ptile(tile, p, n_mblk, e, mb, tt);
      const int rows = min(kPN, __ldg(p.counts + e) - tt * kPN);
      const int n_mma = (rows + 15) & ~15;
      if (!mbar_wait(tfull, acc_phase, abort_flag, p.status, kFlagEpilogue)) break;
      tc_fence_after();
      acc_phase ^= 1u;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c_beg;
      // all loads in flight, then one wait: the accumulator goes back sooner
      uint32_t v[8][16];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c_beg + 16 * c < n_mma) tmem_ld16(tb + 16 * c, v[c]);  // warp-uniform
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader);
      const int64_t row0 = __ldg(p.offsets + e) + (int64_t)tt * kPN + c_beg;
      float* out = p.y + row0 * p.H + mb * kPM + (int)rank * 128 + q * 32 + lane;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c_beg + 16 * c < n_mma) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c_beg + 16 * c + j < rows)
              out[(int64_t)(16 * c + j) * p.H] = __uint_as_float(v[c][j]) * p.acc_scale;
        }
      }
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

}  // namespace

bool nvfp4_pair_supported(const beam_moe_cfg& c) { return c.hidden % kPM == 0; }

cudaError_t launch_down_nvfp4_pair(const beam_moe_cfg& c, const Fp4Layout& F,
                                   const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  const Layout& L = F.base;
  CUtensorMap tw, tx;
  cudaError_t err = encode_tmap_2d_u8(&tw, w.w2_codes, (uint64_t)I / 2, (uint64_t)E * H, 128, 128);
  if (err != cudaSuccess) return err;
  err = encode_tmap_2d_u8(&tx, ws + F.hq, (uint64_t)I / 2, (uint64_t)F.rows, 128, 128);
  if (err != cudaSuccess) return err;
  Pair4Params p;
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.nb_off = reinterpret_cast<const int32_t*>(ws + L.nb_off);
  p.nb2_off = reinterpret_cast<const int32_t*>(ws + L.nb2_off);
  p.w_sf = w.w2_scales;
  p.x_sf = reinterpret_cast<const uint8_t*>(ws + F.hsf);
  p.y = reinterpret_cast<float*>(ws + L.xp);
  p.E = E;
  p.H = H;
  p.nk = I / 256;
  p.sf_chunks = I / 64;
  p.acc_scale = w.w2_scale * w.h_scale;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);

  // Per device: the shared-memory attribute and the number of CTA pairs that
  // can be resident at once. The grid is exactly that many pairs.
  static PerDevice pairs;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P4Cfg::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int resident_pairs = 0;
  err = per_device(pairs, &resident_pairs, [&cfg](int* v) {
    cudaError_t e = cudaFuncSetAttribute(down_nvfp4_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, P4Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t probe = cfg;
    probe.gridDim = dim3((unsigned)(device_sm_count() & ~1));
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, down_nvfp4_pair_kernel, &probe);
    if (e != cudaSuccess) return e;
    if (clusters < 1) return cudaErrorInvalidConfiguration;
    *v = clusters < device_sm_count() / 2 ? clusters : device_sm_count() / 2;
    return cudaSuccess;
  });
  if (err != cudaSuccess) return err;
  cfg.gridDim = dim3((unsigned)(2 * resident_pairs));
  return cudaLaunchKernelEx(&cfg, down_nvfp4_pair_kernel, tw, tx, p);
}

}  // namespace beam
