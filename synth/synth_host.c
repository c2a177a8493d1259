/*
 * synth_host.c - host side of the synthetic input generator (see synth.h).
 * Plain C with OpenMP; every function fills a caller-owned buffer.
 */
#include "synth.h"

#include <stdint.h>

uint64_t synth_stream_key(uint64_t seed, uint64_t stream) {
  return synth_key(seed, stream);
}

uint64_t synth_draw_u64(uint64_t key, uint64_t ctr) { return synth_u64(key, ctr); }

/* out[i] = bf16(N(mu, sigma) deviate number idx0 + i), i < n. */
void synth_host_normal_bf16(uint16_t* out, int64_t n, uint64_t key, uint64_t idx0,
                            float mu, float sigma) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = synth_bf16_bits(synth_normal(key, idx0 + (uint64_t)i, mu, sigma));
}

/* out[i] = N(mu, sigma) deviate number idx0 + i in fp32, i < n. */
void synth_host_normal_f32(float* out, int64_t n, uint64_t key, uint64_t idx0,
                           float mu, float sigma) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = synth_normal(key, idx0 + (uint64_t)i, mu, sigma);
}

/*
 * Activation rows. For each listed row t (rows == NULL: all rows 0..T-1):
 *   x[t][h] = bf16(fmaf(sigma, z(key_x, SYNTH_X_INDEX(attempt[t], t, h)), mu))
 * where mu = 0 when n_centres == 0, else the fp32 centre value
 *   c[t mod n_centres][h] = z(key_c, (t mod n_centres) * H + h).
 * attempts == NULL means attempt 0 for every row.
 */
void synth_host_x_rows(uint16_t* x, int64_t T, int64_t H, uint64_t key_x, uint64_t key_c,
                       int32_t n_centres, float sigma, const int32_t* attempts,
                       const int64_t* rows, int64_t n_rows) {
  int64_t n = rows ? n_rows : T;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n; ++r) {
    int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) continue;
    int32_t a = attempts ? attempts[t] : 0;
    for (int64_t h = 0; h < H; ++h) {
      float mu = 0.0f;
      if (n_centres > 0) mu = synth_z(key_c, (uint64_t)(t % n_centres) * (uint64_t)H + (uint64_t)h);
      x[t * H + h] = synth_bf16_bits(fmaf(sigma, synth_z(key_x, SYNTH_X_INDEX(a, t, h, H)), mu));
    }
  }
}

/* The k indices in [0, n) with the smallest draws synth_u64(key, i), ties to
 * the lower index, written to out[0..k) in ascending index order. Used to pick
 * the biased experts of the skewed workload and the sampled tokens of tests. */
#include <stdlib.h>

typedef struct {
  uint64_t draw;
  int64_t index;
} synth_pair;

static int synth_pair_cmp(const void* a, const void* b) {
  const synth_pair* p = (const synth_pair*)a;
  const synth_pair* q = (const synth_pair*)b;
  if (p->draw != q->draw) return p->draw < q->draw ? -1 : 1;
  return p->index < q->index ? -1 : (p->index > q->index ? 1 : 0);
}

static int synth_index_cmp(const void* a, const void* b) {
  int64_t p = *(const int64_t*)a, q = *(const int64_t*)b;
  return p < q ? -1 : (p > q ? 1 : 0);
}

int synth_host_pick(uint64_t key, int64_t n, int64_t k, int64_t* out) {
  if (k < 0 || k > n) return -1;
  synth_pair* v = (synth_pair*)malloc((size_t)(n > 0 ? n : 1) * sizeof(synth_pair));
  if (!v) return -2;
  for (int64_t i = 0; i < n; ++i) {
    v[i].draw = synth_u64(key, (uint64_t)i);
    v[i].index = i;
  }
  qsort(v, (size_t)n, sizeof(synth_pair), synth_pair_cmp);
  for (int64_t i = 0; i < k; ++i) out[i] = v[i].index;
  free(v);
  qsort(out, (size_t)k, sizeof(int64_t), synth_index_cmp);
  return 0;
}

/* NVFP4 weights of rows [r0, r0 + n) of a matrix with K elements per row:
 * packed codes [n][K/2] and the E4M3 scales row-major [n][K/16] (the device
 * fill writes the same scales in the block-scaled MMA layout instead). */
void synth_host_nvfp4(uint8_t* codes, uint8_t* sf, int64_t r0, int64_t n, int64_t K,
                      uint64_t key) {
#pragma omp parallel for schedule(static)
  for (int64_t r = r0; r < r0 + n; ++r) {
    for (int64_t j = 0; j < K / 2; ++j)
      codes[(r - r0) * (K / 2) + j] = synth_nvfp4_byte(key, (uint64_t)r * (uint64_t)K, (uint64_t)j);
    for (int64_t b = 0; b < K / 16; ++b)
      sf[(r - r0) * (K / 16) + b] = synth_nvfp4_scale(key, (uint64_t)r * (uint64_t)(K / 16) + (uint64_t)b);
  }
}
