/*
 * synth_dev.cu -- GPU fill routines of the synthetic input generator, the
 * device twin of synth_host.c (same header, same bytes). Used to fill
 * multi-gigabyte expert arenas in place. All pointers are device pointers;
 * calls are asynchronous on the given stream and return 0 on success, 1 on a
 * bad argument and 2 on a launch error.
 */
#include <cuda_runtime.h>
#include "synth_gen.h"

namespace {

__global__ void k_codes(uint64_t key, int bits, int64_t first, int64_t n, uint8_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = syn_code(key, (uint64_t)(first + i), bits);
}

__global__ void k_uniform_bf16(uint64_t key, float lo, float span, int64_t first, int64_t n, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = syn_bf16_rne(syn_uniform(key, (uint64_t)(first + i), lo, span));
}

__global__ void k_normal_bf16(uint64_t key, float sigma, int64_t first, int64_t n, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = syn_bf16_rne(syn_normal(key, (uint64_t)(first + i), sigma));
}

__global__ void k_normal_f32(uint64_t key, float sigma, int64_t first, int64_t n, float* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = syn_normal(key, (uint64_t)(first + i), sigma);
}

inline unsigned grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return (unsigned)g;
}

inline int launched() { return cudaGetLastError() == cudaSuccess ? 0 : 2; }

}  // namespace

extern "C" {

int syn_fill_codes_dev(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d, int bits,
                       int64_t first, int64_t n, uint8_t* out, void* stream) {
  if (!out || n < 0 || first < 0 || bits < 1 || bits > 8) return 1;
  if (n == 0) return 0;
  k_codes<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, a, b, c, d), bits, first, n, out);
  return launched();
}

int syn_fill_uniform_bf16_dev(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d, float lo,
                              float span, int64_t first, int64_t n, uint16_t* out, void* stream) {
  if (!out || n < 0 || first < 0) return 1;
  if (n == 0) return 0;
  k_uniform_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, a, b, c, d), lo, span, first, n, out);
  return launched();
}

int syn_fill_normal_bf16_dev(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d, float sigma,
                             int64_t first, int64_t n, uint16_t* out, void* stream) {
  if (!out || n < 0 || first < 0) return 1;
  if (n == 0) return 0;
  k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, a, b, c, d), sigma, first, n, out);
  return launched();
}

int syn_fill_normal_f32_dev(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d, float sigma,
                            int64_t first, int64_t n, float* out, void* stream) {
  if (!out || n < 0 || first < 0) return 1;
  if (n == 0) return 0;
  k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, a, b, c, d), sigma, first, n, out);
  return launched();
}

}  // extern "C"
