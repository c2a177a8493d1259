// nvfp4.cu - the Beam MoE block with NVFP4 experts and NVFP4 activations
// (W4A4): the 4-bit format the launch post "Welcome Beam" names for Blackwell
// deployment (section "Mixture of Experts": the NVFP4 checkpoint stores most
// parameters in 4-bit precision for NVIDIA Blackwell GPUs), with E2M1 values,
// one FP8 E4M3 scale per 16 elements along K and one FP32 scale per tensor.
//
// Routing is the same as the bf16 path. Then:
//   permute  quantises each token's x once (per 16 elements: scale =
//            e4m3(amax / (6 g_x)), code = e2m1(x / (scale g_x))) and writes
//            its K copies into expert segments that start on a 128-row
//            boundary, so that a 128-row token tile is exactly one group of
//            scale atoms;
//   gate/up  D = (W13 x) on kind::mxf4nvf4 tensor cores (block scales applied
//            by the MMA from TMEM), times g_w g_x in the epilogue; h =
//            silu(g) u in FP32, quantised the same way with g_h (a 16-element
//            block of h spans 16 TMEM lanes of a warp: shuffles find its
//            maximum) and written as codes + scales;
//   down     y = (W2 h) g_w2 g_h in FP32, then the bf16 path's combine.
//
// Scale factors of a 128-row x 64-element block are a 512-byte atom (row
// r0 + 32 r1, block kb at byte 16 r0 + 4 r1 + kb); atoms of a matrix are
// ordered (row block, 64-element chunk) with the chunk fastest. An atom is
// copied to 4 TMEM columns with tcgen05.cp and named in the MMA.
#include <cuda_bf16.h>

#include "grouped_gemm.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "sm100_fp4.cuh"

namespace beam {
namespace {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBN = 128;          // token rows per tile; expert segments align to it
constexpr int kKB = 256;          // FP4 elements of K per pipeline stage (128 bytes)
constexpr int kCodeTile = 128 * 128;  // bytes of one 128-row x 256-element code tile
constexpr int kSfStage = 4 * 512;     // scale atoms of one 128-row x 256-element tile

__device__ __forceinline__ size_t sf_offset(int64_t r, int64_t b, int64_t K) {
  const int64_t rr = r & 127;
  return (size_t)(((r >> 7) * (K >> 6) + (b >> 2)) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 +
                  (b & 3));
}

// Quantise 16 consecutive values: scale byte and 8 packed code bytes. Every
// step in FP32 with IEEE division; conversions round to nearest, ties to even,
// saturating.
__device__ __forceinline__ uint32_t quantize16(const float (&v)[16], float g, uint2& packed) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t s8 = cvt_e4m3(amax / (6.0f * g));
  const float d = e4m3_to_f32(s8) * g;
  uint32_t w[2] = {0u, 0u};
  if (s8) {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 3] |= cvt_e2m1(v[i] / d) << (4 * (i & 7));
  }
  packed = make_uint2(w[0], w[1]);
  return s8;
}

__global__ void __launch_bounds__(256) quantize_rows_kernel(const float* __restrict__ v,
                                                            int64_t rows, int64_t K, float g,
                                                            uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ sf) {
  const int64_t nb = rows * (K / 16);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb;
       i += (int64_t)gridDim.x * blockDim.x) {
    float x[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) x[j] = v[i * 16 + j];
    uint2 p;
    sf[i] = (uint8_t)quantize16(x, g, p);
    *reinterpret_cast<uint2*>(codes + i * 8) = p;
  }
}

// One CTA per token: rows of its K assignments (unpadded, for the combine) and
// padded rows of the quantised copies.
__global__ void __launch_bounds__(128) permute_nvfp4_kernel(
    const uint16_t* __restrict__ x, int H, int K, int E, const int32_t* __restrict__ ids,
    const int32_t* __restrict__ chunk_base, const uint32_t* __restrict__ chunk_mask,
    const int32_t* __restrict__ offsets, const int32_t* __restrict__ nb_off,
    int32_t* __restrict__ pos, uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf, float gx) {
  __shared__ int s_q[32];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < K) {
    const int e = ids[(size_t)t * K + tid];
    int p = -1, qp = -1;
    if (e >= 0 && e < E) {
      const int c = t / kChunk, tl = t - c * kChunk;
      const uint32_t* m = chunk_mask + ((size_t)c * E + e) * kChunkWords;
      int rank = 0;
      for (int wd = 0; wd < (tl >> 5); ++wd) rank += __popc(m[wd]);
      rank += __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
      p = chunk_base[(size_t)c * E + e] + rank;
      qp = p - offsets[e] + nb_off[e] * kBN;
    }
    s_q[tid] = qp;
    if (blockIdx.y == 0) pos[(size_t)t * K + tid] = p;
  }
  __syncthreads();
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * H);
  for (int b = blockIdx.y * 128 + tid; b < H / 16; b += gridDim.y * 128) {  // this CTA's slice
    const uint4 a = __ldg(src + 2 * b), c = __ldg(src + 2 * b + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
    uint2 packed;
    const uint32_t s8 = quantize16(v, gx, packed);
    for (int k = 0; k < K; ++k) {
      const int qp = s_q[k];
      if (qp < 0) continue;
      *reinterpret_cast<uint2*>(xq + (size_t)qp * (H / 2) + b * 8) = packed;
      xsf[sf_offset(qp, b, H)] = (uint8_t)s8;
    }
  }
}

struct Fp4Params {
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* nb_off;   // prefix of 128-row token blocks per expert
  const int32_t* tile_off; // prefix of token tiles per expert (of the kernel's tile height)
  const uint8_t* w_sf;  // weight scales, atom layout over the stacked weight rows
  const uint8_t* x_sf;  // activation scales, atom layout over the padded rows
  void* out;            // gate/up: h codes [padded rows][I/2]; down: y fp32 [A][H]
  uint8_t* out_sf;      // gate/up: h scales, atom layout over the padded rows (K = I)
  int64_t out_ld;       // gate/up: I / 2 bytes; down: H floats
  int E;
  int nk;               // K / 256
  int Kel;              // K in elements
  int w_rows;           // weight rows per expert (2I or H)
  int up_rows;          // up rows' offset inside an expert (I)
  int n_mblk;           // 128-row weight blocks per expert (I / 128 or H / 128)
  float acc_scale;      // weight tensor scale x activation tensor scale
  float h_scale;        // gate/up: tensor scale of the quantised h
  int I;                // gate/up: intermediate size
  unsigned* status;
};

// Tile -> (expert, 128-row weight block, token tile of the expert); token tiles
// are fastest, so CTAs running at the same time share weight blocks in L2.
__device__ __forceinline__ void decode_tile4(int tile, const Fp4Params& p, int& e, int& mb,
                                             int& tt, int& ntt) {
  int lo = 0, hi = p.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.tile_off + mid) * p.n_mblk <= tile) lo = mid;
    else hi = mid - 1;
  }
  e = lo;
  const int base = __ldg(p.tile_off + e);
  ntt = __ldg(p.tile_off + e + 1) - base;
  const int local = tile - base * p.n_mblk;
  mb = local / ntt;
  tt = local - mb * ntt;
}

template <bool GATEUP>
struct Cfg4 {
  // warp 0 TMA producer, warp 1 MMA issuer, warps 2-3 scale copiers, then the
  // epilogue warps. The MMA issuer issues nothing but MMAs: a tcgen05.cp
  // costs its issuing thread about as long as an MMA, so the scale copies
  // run from two other warps and overlap the MMAs. The gate/up epilogue
  // (SwiGLU + NVFP4 quantisation of h) is the heavy one: two warps per TMEM
  // lane quarter, each on half of the token columns, and its single
  // accumulator is handed back as soon as it is read. The down epilogue only
  // scales and stores y; it has one warp per lane quarter and a second
  // accumulator stage instead.
  static constexpr int kEpiWarps = GATEUP ? 8 : 4;
  static constexpr int kFirstEpiWarp = 4;
  static constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
  static constexpr int kNA = GATEUP ? 2 : 1;   // 128-row A tiles (gate and up, or down)
  static constexpr int kTok = 128;             // token rows per tile (MMA N)
  static constexpr int kTB = kTok / 128;       // 128-row token blocks per tile
  static constexpr int kStageBytes = (kNA + kTB) * (kCodeTile + kSfStage);
  static constexpr int kStagesRaw = (220 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kAccCols = kNA * kTok;  // FP32 accumulator columns per tile
  static constexpr int kAccStages = GATEUP ? 1 : 2;
  // Scale columns per stage: 4 per 64-element chunk and 128-row block. Stage
  // i uses scale buffer i mod kSfBufs, rewritten only after the MMAs of stage
  // i - kSfBufs completed. gate/up keeps two buffers so that 128 TMEM columns
  // are left to park h (FP32, one column per token) between forming it and
  // quantising it: the accumulator is then free for the next tile, and the
  // quantisation runs from TMEM 16 columns at a time with few live registers.
  static constexpr int kSfColsA = 16 * kNA;
  static constexpr int kSfCols = kSfColsA + 16 * kTB;
  static constexpr int kSfBufs = GATEUP ? 2 : kStages;
  static constexpr int kParkCols = GATEUP ? kTok : 0;
  static constexpr int kTmemCols = 512;
  // gate/up: a 512-byte staging slice per epilogue warp gathers 16 tokens'
  // code bytes (16 x 16) and scale pairs (16 x 2) into wide global stores
  static constexpr int kStageOut = GATEUP ? 512 : 0;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + 256 + kEpiWarps * kStageOut;
  static_assert((3 * kStages + 7) * 8 + 8 <= 256, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  static constexpr int kColsPerWarp = kTok * 4 / kEpiWarps;  // token columns per epilogue warp
  static_assert(kAccStages * kAccCols + kSfBufs * kSfCols + kParkCols <= kTmemCols,
                "TMEM overflow");
  static_assert(kSfBufs <= kStages, "scale buffers");
  static_assert(kStages >= 2, "pipeline too shallow");
  static_assert(kColsPerWarp <= 128, "epilogue registers");
};

template <bool GATEUP>
__global__ void __launch_bounds__(Cfg4<GATEUP>::kThreads, 1)
    grouped_gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tm_w,
                              const __grid_constant__ CUtensorMap tm_x, const Fp4Params p) {
  using C = Cfg4<GATEUP>;
  constexpr int STAGES = C::kStages;
  constexpr int TOK = C::kTok;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // stage: [A codes (x kNA)][B codes (x kTB)][A scales (x kNA)][B scales (x kTB)]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* sfready = empty + STAGES;  // the stage's scales are in TMEM
  uint64_t* tfull = sfready + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;  // [0] MMA issuer, [1] and [2] scale copiers
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfready[s], 2);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * C::kEpiWarps);
    }
    for (int d = 0; d < 3; ++d) mbar_init(&drain[d], 1);
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
  const uint32_t tsf = tmem_base + (uint32_t)(C::kAccStages * C::kAccCols);
  const uint32_t tpark = tsf + (uint32_t)(C::kSfBufs * C::kSfCols);
  const int total = __ldg(p.tile_off + p.E) * p.n_mblk;
  const int sf_chunks = p.Kel / 64;  // scale atoms per 128-row block

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, mb, tt, ntt;
        decode_tile4(tile, p, e, mb, tt, ntt);
        const int wrow = e * p.w_rows + mb * kBM;
        const int qblk = __ldg(p.nb_off + e) + tt * C::kTB;  // first 128-row token block
        const int rows = min(TOK, __ldg(p.counts + e) - tt * TOK);
        const int nbb = (rows + 127) >> 7;                   // token blocks present
        const uint64_t pol_w = ntt == 1 ? pol_stream : pol_keep;
        const uint32_t bytes = (uint32_t)((C::kNA + nbb) * (kCodeTile + kSfStage));
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, kFlagProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* ssf = sa + (C::kNA + C::kTB) * kCodeTile;
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kb * (kKB / 2);  // byte coordinate along K
          tma_load_2d(sa, &tm_w, &full[stage], kx, wrow, pol_w);
          bulk_load(ssf, p.w_sf + ((size_t)(wrow / kBM) * sf_chunks + kb * 4) * 512, kSfStage,
                    &full[stage], pol_w);
          if (GATEUP) {
            tma_load_2d(sa + kCodeTile, &tm_w, &full[stage], kx, wrow + p.up_rows, pol_w);
            bulk_load(ssf + kSfStage,
                      p.w_sf + ((size_t)((wrow + p.up_rows) / kBM) * sf_chunks + kb * 4) * 512,
                      kSfStage, &full[stage], pol_w);
          }
          for (int b = 0; b < nbb; ++b) {
            tma_load_2d(sa + (C::kNA + b) * kCodeTile, &tm_x, &full[stage], kx,
                        (qblk + b) * 128, pol_keep);
            bulk_load(ssf + (C::kNA + b) * kSfStage,
                      p.x_sf + ((size_t)(qblk + b) * sf_chunks + kb * 4) * 512, kSfStage,
                      &full[stage], pol_keep);
          }
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
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int sfbuf = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, mb, tt, ntt;
        decode_tile4(tile, p, e, mb, tt, ntt);
        const int rows = min(TOK, __ldg(p.counts + e) - tt * TOK);
        const uint32_t n_mma = (uint32_t)((rows + 15) & ~15);
        const uint32_t idesc = idesc_nvf4(kBM, n_mma);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.status, kFlagMma)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * C::kAccCols);
        const uint32_t d1 = d0 + TOK;
        for (int kb = 0; kb < p.nk; ++kb) {
          // operands landed and their scales copied to this stage's columns
          if (!mbar_wait(&sfready[stage], phase, abort_flag, p.status, kFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(smem + stage * C::kStageBytes);
          const uint32_t tsf_s = tsf + (uint32_t)(sfbuf * C::kSfCols);
          const uint32_t tsfb = tsf_s + C::kSfColsA;
          if (++sfbuf == C::kSfBufs) sfbuf = 0;
          const uint64_t da0 = smem_desc_k_sw128(sa);
          const uint64_t da1 = smem_desc_k_sw128(sa + kCodeTile);
          const uint64_t db = smem_desc_k_sw128(sa + C::kNA * kCodeTile);
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // 64 FP4 elements (32 bytes) per MMA
            const uint32_t accum = (kb | j) != 0;
            const uint32_t sfb = tsfb + 4 * C::kTB * j;
            umma_nvf4(d0, da0 + 2u * j, db + 2u * j, idesc, tsf_s + 4 * j, sfb, accum);
            if (GATEUP) umma_nvf4(d1, da1 + 2u * j, db + 2u * j, idesc, tsf_s + 16 + 4 * j, sfb, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == C::kAccStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else if (warp < C::kFirstEpiWarp) {
    if (lane == 0) {
      // ------------------------------------------------------ scale copiers
      // Warp 2 copies chunks 0-1 of every operand's scales, warp 3 chunks
      // 2-3, into the stage's TMEM columns: chunk j of the A tile(s) at 4j
      // (gate or down) and 16 + 4j (up), chunk j of token block b at
      // kSfColsA + 4 (kTB j + b), so that a 256-row B operand would find rows
      // 128-255 in the four columns after rows 0-127. Each commits to the
      // stage's sfready barrier, which completes when both warps' copies have.
      const int j0 = 2 * (warp - 2);
      const int64_t ntiles = total > (int)blockIdx.x ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
      const int64_t nstages = ntiles * p.nk;
      int stage = 0;
      uint32_t phase = 0;
      int sfbuf = 0;
      for (int64_t i = 0; i < nstages; ++i) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.status, kFlagMma)) break;
        if (C::kSfBufs < STAGES && i >= C::kSfBufs) {
          // the MMAs of stage i - kSfBufs, which read this buffer, are done
          const int64_t k = i - C::kSfBufs;
          if (!mbar_wait(&empty[k % STAGES], (uint32_t)((k / STAGES) & 1), abort_flag, p.status,
                         kFlagMma))
            break;
        }
        tc_fence_after();
        const uint32_t ssf = smem_addr(smem + stage * C::kStageBytes) + (C::kNA + C::kTB) * kCodeTile;
        const uint32_t tsf_s = tsf + (uint32_t)(sfbuf * C::kSfCols);
        if (++sfbuf == C::kSfBufs) sfbuf = 0;
        const uint32_t tsfb = tsf_s + C::kSfColsA;
#pragma unroll
        for (int j = j0; j < j0 + 2; ++j) {
          tmem_cp_sf_atom(tsf_s + 4 * j, smem_desc_sf_atom(ssf + 512 * j));
          if (GATEUP) tmem_cp_sf_atom(tsf_s + 16 + 4 * j, smem_desc_sf_atom(ssf + kSfStage + 512 * j));
#pragma unroll
          for (int b = 0; b < C::kTB; ++b)  // an absent second block copies stale bytes
            tmem_cp_sf_atom(tsfb + 4 * (C::kTB * j + b),
                            smem_desc_sf_atom(ssf + (C::kNA + b) * kSfStage + 512 * j));
        }
        umma_commit(&sfready[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      uint64_t* own = &drain[1 + (warp - 2)];
      umma_commit(own);  // this warp's copies are done before TMEM is freed
      mbar_wait(own, 0, nullptr, nullptr, 0u, 100000000ull);
    }
    __syncwarp();
  } else {
    // -------------------------------------------------------------- epilogue
    // Each warp owns TMEM lane quarter q (32 weight rows) and token columns
    // [c_beg, c_beg + HALF) of every tile.
    constexpr int HALF = C::kColsPerWarp;
    const int q = warp & 3;
    const int r = q * 32 + lane;  // weight row inside the 128-row tile
    const int c_beg = ((warp - C::kFirstEpiWarp) >> 2) * HALF;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, mb, tt, ntt;
      decode_tile4(tile, p, e, mb, tt, ntt);
      const int rows = min(TOK, __ldg(p.counts + e) - tt * TOK);
      const int n_mma = (rows + 15) & ~15;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, kFlagEpilogue)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::kAccCols);
      uint64_t* const released = &tempty[acc];
      if (++acc == C::kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (GATEUP) {
        // h = silu(g) u, parked in this warp's TMEM columns; then the
        // accumulator goes back to the MMA warp
        const uint32_t tp = tpark + ((uint32_t)(q * 32) << 16) + (uint32_t)c_beg;
#pragma unroll
        for (int c = 0; c < HALF / 16; ++c) {
          if (c_beg + 16 * c < n_mma) {  // warp-uniform
            uint32_t g[16], u[16], hb[16];
            tmem_ld16(tb + c_beg + 16 * c, g);
            tmem_ld16(tb + TOK + c_beg + 16 * c, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              hb[j] = __float_as_uint(gg::silu_mul(__uint_as_float(g[j]) * p.acc_scale,
                                                   __uint_as_float(u[j]) * p.acc_scale));
            tmem_st16(tp + 16 * c, hb);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(released);

        // This warp's 32 intermediate indices start at i0: 16 code bytes per
        // token, and 2 scale bytes (blocks i0/16 and i0/16 + 1, adjacent in
        // the atom layout) per token.
        const int i0 = mb * kBM + q * 32;
        const int64_t qrow0 = (int64_t)(__ldg(p.nb_off + e) + tt) * kBN;  // 128-row aligned
        uint8_t* hq = static_cast<uint8_t*>(p.out) + qrow0 * p.out_ld + i0 / 2;
        uint8_t* hsf = p.out_sf +
                       ((qrow0 >> 7) * (p.I >> 6) + (i0 >> 6)) * 512 + ((i0 >> 4) & 3);
        uint8_t* so = smem + STAGES * C::kStageBytes + 256 +
                      (warp - C::kFirstEpiWarp) * C::kStageOut;  // [16 tokens][16 B], [16][2 B]
        const float six_g = 6.0f * p.h_scale;
#pragma unroll 2
        for (int c = 0; c < HALF / 16; ++c) {
          if (c_beg + 16 * c < n_mma) {
            uint32_t hb[16];
            tmem_ld16(tp + 16 * c, hb);
            tmem_ld_wait();
            // Codes and scales of 16 tokens first, with no control flow, so
            // that their shuffle and conversion chains overlap; then the
            // stores. Tokens from `rows` up to the 16-row boundary land in
            // the padding of this expert's 128-row segment, which no
            // consumer reads, so they need no guard.
            uint32_t packed[16], scale[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float h = __uint_as_float(hb[j]);
              // 16-element block of h: lanes 0-15 or 16-31 of this warp. The
              // magnitudes' bit patterns order like the values.
              uint32_t am = hb[j] & 0x7FFFFFFFu;
#pragma unroll
              for (int off = 1; off < 16; off <<= 1)
                am = max(am, __shfl_xor_sync(0xffffffffu, am, off));
              const uint32_t s8 = cvt_e4m3(__fdividef(__uint_as_float(am), six_g));
              const float d = e4m3_to_f32(s8) * p.h_scale;
              const uint32_t code = s8 ? cvt_e2m1(__fdividef(h, d)) : 0u;
              packed[j] = code | (__shfl_xor_sync(0xffffffffu, code, 1) << 4);
              scale[j] = s8;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if ((lane & 1) == 0) so[16 * j + (lane >> 1)] = (uint8_t)packed[j];
              if ((lane & 15) == 0) so[256 + 2 * j + (lane >> 4)] = (uint8_t)scale[j];
            }
            __syncwarp();
            if (lane < 16) {  // token t = c_beg + 16 c + lane
              const int t = c_beg + 16 * c + lane;
              *reinterpret_cast<uint4*>(hq + t * p.out_ld) =
                  *reinterpret_cast<const uint4*>(so + 16 * lane);
              *reinterpret_cast<uint16_t*>(hsf + (t & 31) * 16 + (t >> 5) * 4) =
                  *reinterpret_cast<const uint16_t*>(so + 256 + 2 * lane);
            }
            __syncwarp();
          }
        }
      } else {
        // y = acc x scale straight from TMEM; the second accumulator stage
        // keeps the MMA warp busy meanwhile
        const int64_t row0 = __ldg(p.offsets + e) + (int64_t)tt * TOK;
        float* out = static_cast<float*>(p.out) + (row0 + c_beg) * p.out_ld + mb * kBM + r;
        for (int c0 = 0; c0 < HALF && c_beg + c0 < n_mma; c0 += 16) {
          uint32_t y[16];
          tmem_ld16(tb + c_beg + c0, y);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c_beg + c0 + j < rows) out[(c0 + j) * p.out_ld] = __uint_as_float(y[j]) * p.acc_scale;
        }
        tc_fence_before();
        mbar_arrive(released);
      }
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

template <bool GATEUP>
cudaError_t run4(const CUtensorMap& tw, const CUtensorMap& tx, const Fp4Params& p,
                 cudaStream_t st) {
  using C = Cfg4<GATEUP>;
  static PerDevice configured;  // the shared-memory attribute, once per device
  int unused = 0;
  cudaError_t err = per_device(configured, &unused, [](int*) {
    return cudaFuncSetAttribute(grouped_gemm_nvfp4_kernel<GATEUP>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (err != cudaSuccess) return err;
  grouped_gemm_nvfp4_kernel<GATEUP><<<device_sm_count(), C::kThreads, C::kSmemBytes, st>>>(tw, tx, p);
  return cudaGetLastError();
}

// 2-D byte tensor [rows][cols bytes], box {128 bytes, 128 rows}, 128-byte swizzle.
cudaError_t encode_codes_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  return encode_tmap_2d_u8(map, base, cols, rows, 128, 128);
}

}  // namespace

Fp4Layout make_layout_nvfp4(const beam_moe_cfg& c, int64_t T, int sms) {
  Fp4Layout F;
  F.base = make_layout(c, T, sms);
  Layout& L = F.base;
  L.bn = kBN;  // token tiles of 128 rows; expert segments padded to them
  L.pair_gateup = L.pair_down = 0;
  L.light_max = 0;
  // CTA pairs for the down GEMM once experts average 1024 rows or more. A
  // pair tile of 256 weight rows x 256 tokens halves the operand bytes per
  // FLOP, but its one 256-column accumulator leaves the MMAs idle while the
  // epilogue drains it; measured, it wins only at the largest batches
  // (T = 65536: 5.46 against 5.90 ms; T = 4096: 0.553 against 0.536 ms).
  F.pair_down = ((double)T * c.top_k / c.n_experts >= 1024.0 && nvfp4_pair_supported(c)) ? 1 : 0;
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  F.rows = ((L.A + kBN - 1) / kBN + E) * (int64_t)kBN;  // bound on the padded rows
  size_t o = L.route_end;
  auto take = [&](size_t bytes, size_t align) {
    o = (o + align - 1) / align * align;
    size_t at = o;
    o += bytes;
    return at;
  };
  F.xq = take((size_t)F.rows * H / 2, 1024);
  F.xsf = take((size_t)F.rows * H / 16, 1024);
  F.hq = take((size_t)F.rows * I / 2, 1024);
  F.hsf = take((size_t)F.rows * I / 16, 1024);
  L.xp = take((size_t)L.A * H * 4, 1024);  // fp32 y, read by the combine
  L.h = 0;
  L.total = (o + 255) / 256 * 256;
  return F;
}

bool nvfp4_supported(const beam_moe_cfg& c) {
  return c.hidden % kKB == 0 && c.inter % kKB == 0;
}

cudaError_t launch_permute_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F, const uint16_t* x,
                                 float gx, char* ws, cudaStream_t st) {
  const Layout& L = F.base;
  permute_nvfp4_kernel<<<dim3((unsigned)L.T, (unsigned)h_slices(L.T, c.hidden / 16)), 128, 0, st>>>(
      x, c.hidden, c.top_k, c.n_experts, reinterpret_cast<const int32_t*>(ws + L.ids),
      reinterpret_cast<const int32_t*>(ws + L.chunk_cnt),
      reinterpret_cast<const uint32_t*>(ws + L.chunk_mask),
      reinterpret_cast<const int32_t*>(ws + L.offsets),
      reinterpret_cast<const int32_t*>(ws + L.nb_off), reinterpret_cast<int32_t*>(ws + L.pos),
      reinterpret_cast<uint8_t*>(ws + F.xq), reinterpret_cast<uint8_t*>(ws + F.xsf), gx);
  return cudaGetLastError();
}

static Fp4Params base_params4(const beam_moe_cfg& c, const Fp4Layout& F, char* ws) {
  const Layout& L = F.base;
  Fp4Params p;
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.nb_off = reinterpret_cast<const int32_t*>(ws + L.nb_off);
  p.tile_off = p.nb_off;
  p.E = c.n_experts;
  p.status = reinterpret_cast<unsigned*>(ws + L.status);
  p.I = c.inter;
  return p;
}

cudaError_t launch_gateup_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F,
                                const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  Fp4Params p = base_params4(c, F, ws);
  CUtensorMap tw, tx;
  cudaError_t err = encode_codes_map(&tw, w.w13_codes, (uint64_t)H / 2, (uint64_t)E * 2 * I);
  if (err != cudaSuccess) return err;
  err = encode_codes_map(&tx, ws + F.xq, (uint64_t)H / 2, (uint64_t)F.rows);
  if (err != cudaSuccess) return err;
  p.w_sf = w.w13_scales;
  p.x_sf = reinterpret_cast<const uint8_t*>(ws + F.xsf);
  p.out = ws + F.hq;
  p.out_sf = reinterpret_cast<uint8_t*>(ws + F.hsf);
  p.out_ld = I / 2;
  p.nk = H / kKB;
  p.Kel = H;
  p.w_rows = 2 * I;
  p.up_rows = I;
  p.n_mblk = I / kBM;
  p.acc_scale = w.w13_scale * w.x_scale;
  p.h_scale = w.h_scale;
  return run4<true>(tw, tx, p, st);
}

cudaError_t launch_down_nvfp4(const beam_moe_cfg& c, const Fp4Layout& F,
                              const beam_moe_nvfp4_experts& w, char* ws, cudaStream_t st) {
  const int H = c.hidden, I = c.inter, E = c.n_experts;
  Fp4Params p = base_params4(c, F, ws);
  CUtensorMap tw, tx;
  cudaError_t err = encode_codes_map(&tw, w.w2_codes, (uint64_t)I / 2, (uint64_t)E * H);
  if (err != cudaSuccess) return err;
  err = encode_codes_map(&tx, ws + F.hq, (uint64_t)I / 2, (uint64_t)F.rows);
  if (err != cudaSuccess) return err;
  if (Cfg4<false>::kTok == 256)  // token tiles of two 128-row blocks
    p.tile_off = reinterpret_cast<const int32_t*>(ws + F.base.nb2_off);
  p.w_sf = w.w2_scales;
  p.x_sf = reinterpret_cast<const uint8_t*>(ws + F.hsf);
  p.out = ws + F.base.xp;
  p.out_sf = nullptr;
  p.out_ld = H;
  p.nk = I / kKB;
  p.Kel = I;
  p.w_rows = H;
  p.up_rows = 0;
  p.n_mblk = H / kBM;
  p.acc_scale = w.w2_scale * w.h_scale;
  p.h_scale = w.h_scale;
  return run4<false>(tw, tx, p, st);
}

cudaError_t launch_quantize_rows(int64_t rows, int64_t K, const float* v, float g, uint8_t* codes,
                                 uint8_t* sf, cudaStream_t st) {
  const int64_t nb = rows * (K / 16);
  const int64_t grid = (nb + 255) / 256 < 148 * 8 ? (nb + 255) / 256 : 148 * 8;
  quantize_rows_kernel<<<(unsigned)(grid > 0 ? grid : 1), 256, 0, st>>>(v, rows, K, g, codes, sf);
  return cudaGetLastError();
}

}  // namespace beam
