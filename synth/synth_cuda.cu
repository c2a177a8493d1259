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

}  // extern "C"
