// sm100_fp4.cuh - inline-PTX wrappers for block-scaled FP4 (NVFP4) on sm_100a:
// 1-D bulk copies, scale atoms copied to TMEM (tcgen05.cp), the kind::mxf4nvf4
// MMA, and the E4M3 / E2M1 conversions. Encodings follow the PTX ISA.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace beam {

// ----------------------------------------------------- block-scaled FP4
// 1-D bulk copy global -> shared (sizes and addresses multiples of 16 bytes).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Shared-memory descriptor of a 512-byte scale atom (32 rows of 16 bytes,
// no swizzle: 8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sf_atom(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;             // leading byte offset (one 16-byte column: unused)
  d |= (uint64_t)(128u >> 4) << 32;    // stride byte offset: 8 rows x 16 bytes
  d |= (uint64_t)1u << 46;             // descriptor version for tcgen05
  return d;                            // layout type 0: no swizzle
}

// Copy one scale atom to TMEM: 32 lanes x 128 bits, replicated to all four
// lane quadrants (4 columns starting at taddr).
__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B, E4M3 scales, K-major.
__device__ __forceinline__ uint32_t idesc_nvf4(uint32_t M, uint32_t N) {
  return (1u << 7)            // A format E2M1
         | (1u << 10)         // B format E2M1
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16 (scale format bit 23 = 0: E4M3)
}

// D (+)= (A * SFA) (B * SFB)^T, 64 FP4 elements of K, 16-element scale blocks.
__device__ __forceinline__ void umma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Block-scaled FP4 MMA over a CTA pair (M = 256: 128 rows of A from each
// CTA; B split by N halves), issued by one thread of the even CTA. Each CTA
// reads the scales of its own A rows and of all N B rows from its own TMEM
// at the given columns.
__device__ __forceinline__ void umma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Arrive once on the mbarrier at this shared-memory offset in every CTA of
// `cta_mask` when this thread's earlier tcgen05 operations (its scale copies)
// are done.
__device__ __forceinline__ void tc_commit_to(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_addr(bar)),
      "h"(cta_mask)
      : "memory");
}

// TMEM store, 32 lanes x 32 bits, 16 consecutive columns (this warp's lane quarter).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// FP32 -> E4M3 byte (nearest, ties to even, saturating at 448).
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(v));
  return r & 0xFFu;
}

// FP32 -> E2M1 code (nearest, ties to even, saturating at 6), low 4 bits.
__device__ __forceinline__ uint32_t cvt_e2m1(float v) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(v));
  return r & 0xFu;
}

// E4M3 byte (non-negative, finite) -> FP32, exact.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  // hardware E4M3 -> F16 conversion of the byte pair (b, 0); the zero byte
  // converts to +0, so OR-ing the halves picks b's value in either order
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(b & 0xFFu)));
  return __half2float(__ushort_as_half((uint16_t)((h2 | (h2 >> 16)) & 0xFFFFu)));
}

}  // namespace beam
