// combine.cuh -- moe_combine_residual: weighted combine of the routed experts
// with the shared expert and the residual, optional shared-expert sigmoid
// gate, optional RMSNorm'd bf16 copy for the next layer (Flash-MoE page,
// sections "Metal Compute Shaders" and "Deferred GPU Expert Compute").
#pragma once

#include "common.cuh"

namespace moeq {

constexpr int kCombineThreads = 512;

struct CombineParams {
  const float* y;          // [B, K+1, H]
  const float* w;          // [B, K]
  const uint16_t* x;       // [B, H] bf16
  const float* resid_in;   // [B, H] or null (then r = x)
  const uint16_t* gate_w;  // [H] bf16 or null (gamma = 1)
  float* resid_out;        // [B, H]
  uint16_t* xnorm;         // [B, H] bf16 or null
  int B, H, K;
  float eps;
};

// grid: B CTAs, one token each.
__global__ void __launch_bounds__(kCombineThreads) k_combine(CombineParams p) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  pdl_wait();
  const uint16_t* xb = p.x + (size_t)b * p.H;
  float gamma = 1.f;
  if (p.gate_w) {
    float a = 0.f;
    for (int j = threadIdx.x; j < p.H; j += blockDim.x)
      a += bf16_bits_to_f32(p.gate_w[j]) * bf16_bits_to_f32(xb[j]);
    a = block_sum(a, red);
    gamma = 1.f / (1.f + expf(-a));
  }
  float wk[MOEQ_MAX_K];
#pragma unroll
  for (int k = 0; k < MOEQ_MAX_K; ++k) wk[k] = k < p.K ? p.w[(size_t)b * p.K + k] : 0.f;
  const float* yb = p.y + (size_t)b * (p.K + 1) * p.H;
  float ss = 0.f;
  constexpr int U = 4;  // elements per thread in flight
  for (int j0 = threadIdx.x; j0 < p.H; j0 += blockDim.x * U) {
    float acc[U], ys[U][MOEQ_MAX_K + 1];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * blockDim.x;
      if (j < p.H) {
        acc[u] = p.resid_in ? p.resid_in[(size_t)b * p.H + j] : bf16_bits_to_f32(xb[j]);
#pragma unroll
        for (int k = 0; k <= MOEQ_MAX_K; ++k)
          if (k <= p.K) ys[u][k] = yb[(size_t)k * p.H + j];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * blockDim.x;
      if (j < p.H) {
        float a = acc[u];
#pragma unroll
        for (int k = 0; k < MOEQ_MAX_K; ++k)
          if (k < p.K) a += wk[k] * ys[u][k];
        a += gamma * ys[u][p.K];
        p.resid_out[(size_t)b * p.H + j] = a;
        ss += a * a;
      }
    }
  }
  if (p.xnorm) {
    ss = block_sum(ss, red);
    const float inv = rsqrtf(ss / (float)p.H + p.eps);
    // each thread re-reads only the elements it wrote itself
    for (int j = threadIdx.x; j < p.H; j += blockDim.x)
      p.xnorm[(size_t)b * p.H + j] = f32_to_bf16_bits(p.resid_out[(size_t)b * p.H + j] * inv);
  }
  pdl_trigger();
}

}  // namespace moeq
