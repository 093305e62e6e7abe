/*
 * synth_gen.h -- seeded, counter-based generator of synthetic inputs.
 *
 * This header is input-generation infrastructure shared by the test harness,
 * the oracle's callers and the benchmark. It holds none of the MoE method's
 * arithmetic: it only turns (seed, tuple, element index) into codes, scales,
 * biases, activations and router weights with stated distributions. The same
 * source compiles for the host (synth_host.c) and for the GPU (synth_dev.cu),
 * so a tensor generated on either side is byte-identical.
 *
 * Generator: the SplitMix64 output function (G. Steele, D. Lea, C. Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014), used in
 * counter mode: draw(key, i) = mix64(key + GOLDEN * (i + 1)).
 *
 * Distributions (all integer work, plus IEEE fp32 multiply and add done one
 * rounded operation at a time, never contracted into an fma):
 *   code     b-bit unsigned:   draw & (2^b - 1)
 *   uniform  lo + span * t,    t = (draw >> 40) * 2^-24   (24-bit grid on [0,1))
 *   normal   sigma * z,        z = (S - 393210) * 2^-16, S = sum of twelve
 *            16-bit fields of three consecutive draws (Irwin-Hall of order 12,
 *            mean 0 and variance ~1: a stand-in for N(0,1))
 * bf16 results are rounded to nearest-even from the fp32 value.
 */
#ifndef SYNTH_GEN_H
#define SYNTH_GEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_HD __host__ __device__ __forceinline__
#else
#define SYN_HD static inline
#endif

#define SYN_GOLDEN 0x9E3779B97F4A7C15ull

/* tensor tags used in the key tuple */
enum {
  SYN_TAG_CODES = 1,   /* matrix = 0 gate, 1 up, 2 down */
  SYN_TAG_SCALE = 2,
  SYN_TAG_BIAS = 3,
  SYN_TAG_ROUTER = 4,
  SYN_TAG_X = 5,
  SYN_TAG_SHARED_GATE = 6,
  SYN_TAG_RESID = 7
};

SYN_HD uint64_t syn_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* key of one tensor: folds (seed, a, b, c, d) through the mixer */
SYN_HD uint64_t syn_key(uint64_t seed, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  uint64_t h = syn_mix64(seed + SYN_GOLDEN);
  h = syn_mix64(h + SYN_GOLDEN * ((uint64_t)a + 1));
  h = syn_mix64(h + SYN_GOLDEN * ((uint64_t)b + 1));
  h = syn_mix64(h + SYN_GOLDEN * ((uint64_t)c + 1));
  h = syn_mix64(h + SYN_GOLDEN * ((uint64_t)d + 1));
  return h;
}

SYN_HD uint64_t syn_draw(uint64_t key, uint64_t i) {
  return syn_mix64(key + SYN_GOLDEN * (i + 1));
}

SYN_HD uint32_t syn_f32_bits(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  union { float f; uint32_t u; } v;
  v.f = f;
  return v.u;
#endif
}

SYN_HD float syn_mul(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  return a * b;
#endif
}

SYN_HD float syn_add(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs only) */
SYN_HD uint16_t syn_bf16_rne(float f) {
  uint32_t u = syn_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

SYN_HD uint8_t syn_code(uint64_t key, uint64_t i, int bits) {
  return (uint8_t)(syn_draw(key, i) & ((1ull << bits) - 1ull));
}

SYN_HD float syn_uniform(uint64_t key, uint64_t i, float lo, float span) {
  uint32_t u = (uint32_t)(syn_draw(key, i) >> 40);
  float t = syn_mul((float)u, 5.9604644775390625e-08f); /* 2^-24, exact */
  return syn_add(lo, syn_mul(span, t));
}

SYN_HD float syn_normal(uint64_t key, uint64_t i, float sigma) {
  uint32_t s = 0;
  for (int k = 0; k < 3; ++k) {
    uint64_t r = syn_draw(key, 3 * i + (uint64_t)k);
    s += (uint32_t)(r & 0xFFFF) + (uint32_t)((r >> 16) & 0xFFFF) +
         (uint32_t)((r >> 32) & 0xFFFF) + (uint32_t)(r >> 48);
  }
  int32_t t = (int32_t)s - 393210;
  float z = syn_mul((float)t, 1.52587890625e-05f); /* 2^-16, exact */
  return syn_mul(sigma, z);
}

#endif /* SYNTH_GEN_H */
