/*
 * synth_host.c -- host (CPU) fill routines of the synthetic input generator.
 * Element i of a tensor depends only on (seed, tuple, i); see synth_gen.h.
 * Build with -ffp-contract=off so that each fp32 multiply and add rounds on
 * its own, exactly as the device copy does.
 */
#include "synth_gen.h"

int syn_fill_codes(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                   int bits, int64_t first, int64_t n, uint8_t* out) {
  if (!out || n < 0 || first < 0 || bits < 1 || bits > 8) return 1;
  uint64_t key = syn_key(seed, a, b, c, d);
  for (int64_t i = 0; i < n; ++i) out[i] = syn_code(key, (uint64_t)(first + i), bits);
  return 0;
}

int syn_fill_uniform_bf16(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                          float lo, float span, int64_t first, int64_t n, uint16_t* out) {
  if (!out || n < 0 || first < 0) return 1;
  uint64_t key = syn_key(seed, a, b, c, d);
  for (int64_t i = 0; i < n; ++i) out[i] = syn_bf16_rne(syn_uniform(key, (uint64_t)(first + i), lo, span));
  return 0;
}

int syn_fill_normal_bf16(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                         float sigma, int64_t first, int64_t n, uint16_t* out) {
  if (!out || n < 0 || first < 0) return 1;
  uint64_t key = syn_key(seed, a, b, c, d);
  for (int64_t i = 0; i < n; ++i) out[i] = syn_bf16_rne(syn_normal(key, (uint64_t)(first + i), sigma));
  return 0;
}

int syn_fill_normal_f32(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                        float sigma, int64_t first, int64_t n, float* out) {
  if (!out || n < 0 || first < 0) return 1;
  uint64_t key = syn_key(seed, a, b, c, d);
  for (int64_t i = 0; i < n; ++i) out[i] = syn_normal(key, (uint64_t)(first + i), sigma);
  return 0;
}
