/*
 * synth_cuda.cu - device side of the synthetic input generator (see synth.h).
 *
 * Fills device buffers with exactly the bytes the host functions in
 * synth_host.c produce for the same arguments, so that multi-GB expert
 * weights need not be generated on the host and copied. Grids are sized as a
 * multiple of the SM count and stride over the buffer.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth.h"

namespace {

__global__ void fill_normal_bf16(uint16_t* out, int64_t n, uint64_t key, uint64_t idx0, float mu,
                                 float sigma) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = synth_bf16_bits(synth_normal(key, idx0 + (uint64_t)i, mu, sigma));
}

__global__ void fill_normal_f32(float* out, int64_t n, uint64_t key, uint64_t idx0, float mu,
                                float sigma) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = synth_normal(key, idx0 + (uint64_t)i, mu, sigma);
}

__global__ void fill_x(uint16_t* x, int64_t T, int64_t H, uint64_t key_x, uint64_t key_c,
                       int32_t n_centres, float sigma, const int32_t* attempts) {
  int64_t n = T * H;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    int64_t t = i / H, h = i - t * H;
    int32_t a = attempts ? attempts[t] : 0;
    float mu = 0.0f;
    if (n_centres > 0) mu = synth_z(key_c, (uint64_t)(t % n_centres) * (uint64_t)H + (uint64_t)h);
    x[i] = synth_bf16_bits(fmaf(sigma, synth_z(key_x, SYNTH_X_INDEX(a, t, h, H)), mu));
  }
}

__global__ void fill_nvfp4_codes(uint8_t* codes, int64_t rows, int64_t K, uint64_t key) {
  const int64_t n = rows * (K / 2);
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t r = i / (K / 2), j = i - r * (K / 2);
    codes[i] = synth_nvfp4_byte(key, (uint64_t)r * (uint64_t)K, (uint64_t)j);
  }
}

__global__ void fill_nvfp4_scales(uint8_t* sf, int64_t rows, int64_t K, uint64_t key) {
  const int64_t n = rows * (K / 16);
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t r = i / (K / 16), b = i - r * (K / 16);
    sf[synth_sf_offset((uint64_t)r, (uint64_t)b, (uint64_t)K)] = synth_nvfp4_scale(key, (uint64_t)i);
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

extern "C" {

/* Each call enqueues one kernel on `stream` and returns the launch status
 * (a cudaError_t value, 0 on success). */
int synth_dev_normal_bf16(void* out, int64_t n, uint64_t key, uint64_t idx0, float mu,
                          float sigma, void* stream) {
  if (n <= 0) return 0;
  fill_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((uint16_t*)out, n, key, idx0,
                                                                  mu, sigma);
  return (int)cudaGetLastError();
}

int synth_dev_normal_f32(void* out, int64_t n, uint64_t key, uint64_t idx0, float mu, float sigma,
                         void* stream) {
  if (n <= 0) return 0;
  fill_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((float*)out, n, key, idx0, mu,
                                                                 sigma);
  return (int)cudaGetLastError();
}

int synth_dev_x(void* x, int64_t T, int64_t H, uint64_t key_x, uint64_t key_c, int32_t n_centres,
                float sigma, const void* attempts, void* stream) {
  if (T * H <= 0) return 0;
  fill_x<<<grid_for(T * H), 256, 0, (cudaStream_t)stream>>>(
      (uint16_t*)x, T, H, key_x, key_c, n_centres, sigma, (const int32_t*)attempts);
  return (int)cudaGetLastError();
}

/* NVFP4 weights of a whole [rows][K] matrix (rows a multiple of 128): packed
 * codes [rows][K/2] and scales in the block-scaled MMA layout. */
int synth_dev_nvfp4(void* codes, void* sf, int64_t rows, int64_t K, uint64_t key, void* stream) {
  if (rows * K <= 0) return 0;
  fill_nvfp4_codes<<<grid_for(rows * K / 2), 256, 0, (cudaStream_t)stream>>>((uint8_t*)codes, rows,
                                                                             K, key);
  fill_nvfp4_scales<<<grid_for(rows * K / 16), 256, 0, (cudaStream_t)stream>>>((uint8_t*)sf, rows,
                                                                               K, key);
  return (int)cudaGetLastError();
}

}  // extern "C"
