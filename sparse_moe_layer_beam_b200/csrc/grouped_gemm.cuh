// grouped_gemm.cuh - pieces shared by the 1-CTA and 2-CTA grouped GEMMs.
#pragma once

#include <cuda_bf16.h>

#include "internal.h"

namespace beam {
namespace gg {

struct GemmParams {
  const int32_t* counts;  // [E] rows routed to each expert
  const int32_t* offsets; // [E + 1] first permuted row of each expert
  const int32_t* nb_off;  // [E + 1] prefix of token blocks per expert
  void* out;              // [A][out_ld] output rows: bf16 h (gate/up), fp32 y (down)
  int64_t out_ld;
  int E;
  int nk;       // K / 64
  int w_rows;   // weight rows per expert (2I or H)
  int up_rows;  // row offset of the up projection inside an expert (I)
  int n_mblk;   // 128-row weight blocks per expert (I / 128 or H / 128)
  unsigned* status;
  const int32_t* arrive;  // [E] or nullptr: rows arrived per expert (expert parallelism);
                          // a tile's rows are loaded once arrive[e] reaches counts[e]
  int* next_tile;         // CTA-pair kernels: the launch's tile counter (zero at launch)
};

__host__ __device__ constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

// Tile -> (expert, weight block, token block). The largest e with
// nb_off[e] * n_mblk <= tile is never an empty expert.
__device__ __forceinline__ void decode_tile(int tile, const GemmParams& p, int& e, int& mb,
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
  mb = local / nblk;
  nb = local - mb * nblk;
}

// silu(g) u in FP32: silu(g) = g / (1 + e^-g) with the hardware exponential
// and an approximate FP32 division, both within a few FP32 ulps, so h =
// silu(g) u is FP32-accurate before it is rounded to bf16 or quantised to
// NVFP4 (the SwiGLU product is FP32 in "Welcome Beam", section "Residual
// Stream"). A cheaper tanh form (relative error 2^-11) moved h across
// rounding and E2M1 quantisation boundaries often enough to show in the
// output. For g below about -88, e^-g overflows to +inf and the quotient is
// -0.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

}  // namespace gg
}  // namespace beam
