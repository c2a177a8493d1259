/*
 * synth.h - seeded synthetic inputs for the Beam MoE block, shared by the CPU
 * oracle tests and the GPU tests.
 *
 * This module holds none of the MoE block's arithmetic. It only turns a seed,
 * a stream id and an element index into a value, the same way on the host and
 * on the device, so that both sides of a parity test read the same bytes.
 *
 * Generator: splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), used as a counter-based generator: output
 * number i of the stream with key k is mix64(k + (i + 1) * GAMMA).
 *
 * Normal deviates: the sum of twelve uniform 16-bit integers, centred and
 * scaled (the Irwin-Hall approximation of N(0,1); variance 1 - 2^-32, support
 * +-6). Every step is integer arithmetic, then one exact int -> float
 * conversion and one multiply by a power of two, so the deviate z is exactly
 * representable in fp32 and identical on host and device. A value
 * N(mu, sigma) is fmaf(sigma, z, mu): one correctly rounded fused
 * multiply-add, identical on both sides. bf16 values are that fp32 value
 * rounded to nearest even.
 */
#ifndef BEAM_SYNTH_H
#define BEAM_SYNTH_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#include <math.h>
#define SYNTH_HD static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ull

/* Stream ids: every tensor draws from its own stream. */
enum {
  SYNTH_STREAM_X = 1,        /* token activations (noise part)          */
  SYNTH_STREAM_WROUTER = 2,  /* router weights                          */
  SYNTH_STREAM_W13 = 3,      /* stacked gate/up expert weights          */
  SYNTH_STREAM_W2 = 4,       /* stacked down expert weights             */
  SYNTH_STREAM_CENTRES = 5,  /* cluster centres of clustered activations */
  SYNTH_STREAM_BIASPICK = 6, /* choice of the biased ("hot") experts     */
  SYNTH_STREAM_SAMPLE = 7    /* choice of sampled tokens in tests/bench  */
};

/* Element index of activation row t, column h, drawn on attempt a. Rows that
 * a test re-draws use a higher attempt; everything else keeps attempt 0. */
#define SYNTH_X_INDEX(a, t, h, H) \
  ((((uint64_t)(a)) << 40) | ((uint64_t)(t) * (uint64_t)(H) + (uint64_t)(h)))

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* Key of stream `stream` under seed `seed`. */
SYNTH_HD uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64(synth_mix64(seed + SYNTH_GAMMA) ^ (stream * SYNTH_GAMMA));
}

/* Output number `ctr` of the stream with key `key`. */
SYNTH_HD uint64_t synth_u64(uint64_t key, uint64_t ctr) {
  return synth_mix64(key + (ctr + 1ull) * SYNTH_GAMMA);
}

/* Approximately standard-normal deviate number `idx`; exactly representable
 * in fp32 (a multiple of 2^-17 with magnitude at most 6). */
SYNTH_HD float synth_z(uint64_t key, uint64_t idx) {
  int32_t s = 0;
  for (int j = 0; j < 3; ++j) {
    uint64_t r = synth_u64(key, 3ull * idx + (uint64_t)j);
    s += (int32_t)(r & 0xFFFFu) + (int32_t)((r >> 16) & 0xFFFFu) +
         (int32_t)((r >> 32) & 0xFFFFu) + (int32_t)((r >> 48) & 0xFFFFu);
  }
  /* 2 * (s - 12 * 32767.5), |d| <= 786420 < 2^24: the conversion is exact. */
  int32_t d = 2 * s - 12 * 65535;
  return (float)d * (1.0f / 131072.0f);
}

/* N(mu, sigma) in fp32: one correctly rounded fused multiply-add. */
SYNTH_HD float synth_normal(uint64_t key, uint64_t idx, float mu, float sigma) {
  return fmaf(sigma, synth_z(key, idx), mu);
}

/* fp32 -> bf16 bits, round to nearest even (inputs are finite). */
SYNTH_HD uint16_t synth_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ NVFP4
 * Synthetic NVFP4 expert weights (4-bit E2M1 values, one FP8 E4M3 scale per
 * 16 consecutive elements of a row, one FP32 scale per tensor), drawn
 * directly in the format: no quantisation arithmetic is involved.
 *  - element code: a standard-normal deviate z, times 2, mapped to the nearest
 *    E2M1 magnitude {0, .5, 1, 1.5, 2, 3, 4, 6} (fixed thresholds; z is a
 *    multiple of 2^-17 so no tie can occur), sign bit 3;
 *  - block scale: E4M3 byte 0x38 + (u mod 8), i.e. 1.0 .. 1.875.
 * With a tensor scale of 2^-7 the values have a standard deviation of about
 * 0.02, like the bf16 experts. */
SYNTH_HD uint8_t synth_e2m1_code(float z) {
  float m = fabsf(z) * 2.0f;
  uint8_t c;
  if (m < 0.25f) c = 0;
  else if (m < 0.75f) c = 1;
  else if (m < 1.25f) c = 2;
  else if (m < 1.75f) c = 3;
  else if (m < 2.5f) c = 4;
  else if (m < 3.5f) c = 5;
  else if (m < 5.0f) c = 6;
  else c = 7;
  return (uint8_t)(c | (z < 0.0f && c != 0 ? 8u : 0u));
}

/* Packed byte j of a weight row: elements 2j (low nibble) and 2j + 1. The
 * element index of the row's first element is `idx_row`. */
SYNTH_HD uint8_t synth_nvfp4_byte(uint64_t key, uint64_t idx_row, uint64_t j) {
  uint8_t lo = synth_e2m1_code(synth_z(key, idx_row + 2 * j));
  uint8_t hi = synth_e2m1_code(synth_z(key, idx_row + 2 * j + 1));
  return (uint8_t)(lo | (hi << 4));
}

/* E4M3 scale byte of the 16-element block `blk` (global block index). */
SYNTH_HD uint8_t synth_nvfp4_scale(uint64_t key, uint64_t blk) {
  return (uint8_t)(0x38u + (uint32_t)(synth_u64(key ^ 0x5CA1Eull, blk) & 7u));
}

/* Byte offset, inside a scale array in the block-scaled MMA layout, of the
 * scale of row r, 16-element block b, for a matrix whose rows hold K
 * elements: 512-byte atoms of 128 rows x 4 blocks, atoms ordered (row block,
 * 64-element chunk) with the chunk fastest; inside an atom, row r0 + 32 r1
 * and block kb sit at byte 16 r0 + 4 r1 + kb. */
SYNTH_HD uint64_t synth_sf_offset(uint64_t r, uint64_t b, uint64_t K) {
  uint64_t atom = (r / 128) * (K / 64) + b / 4;
  uint64_t rr = r % 128;
  return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (b % 4);
}

#endif /* BEAM_SYNTH_H */
