// combine.cuh -- moe_combine_residual: weighted combine of the routed experts
// with the shared expert and the residual, optional shared-expert sigmoid
// gate, optional RMSNorm'd bf16 copy for the next layer (Flash-MoE page,
// sections "Metal Compute Shaders" and "Deferred GPU Expert Compute").
#pragma once

#include "common.cuh"

namespace moeq {

constexpr int kCombineThreads = 512;
constexpr int kCombineU = 8;  // elements per thread per pass (one pass covers H <= 4096)

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

// grid: B CTAs, one token each. A thread keeps the outputs of its first pass
// in registers for the RMSNorm'd copy; only when H > kCombineThreads *
// kCombineU does it read later ones back (each thread only what it wrote).
__global__ void __launch_bounds__(kCombineThreads) k_combine(CombineParams p) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  pdl_trigger();
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
  // weight of slot k: w_k for the routed slots, gamma for the shared one (k == K)
  float wk[MOEQ_MAX_K + 1];
#pragma unroll
  for (int k = 0; k <= MOEQ_MAX_K; ++k) wk[k] = k < p.K ? p.w[(size_t)b * p.K + k] : (k == p.K ? gamma : 0.f);
  const float* yb = p.y + (size_t)b * (p.K + 1) * p.H;
  float* rb = p.resid_out + (size_t)b * p.H;
  float ss = 0.f, keep[kCombineU];
  const int stride = blockDim.x * kCombineU;
  for (int j0 = threadIdx.x; j0 < p.H; j0 += stride) {
    float acc[kCombineU];
#pragma unroll
    for (int u = 0; u < kCombineU; ++u) {
      const int j = j0 + u * blockDim.x;
      acc[u] = j < p.H ? (p.resid_in ? p.resid_in[(size_t)b * p.H + j] : bf16_bits_to_f32(xb[j])) : 0.f;
    }
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_K; ++k) {
      if (k <= p.K) {
#pragma unroll
        for (int u = 0; u < kCombineU; ++u) {
          const int j = j0 + u * blockDim.x;
          if (j < p.H) acc[u] += wk[k] * yb[(size_t)k * p.H + j];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kCombineU; ++u) {
      const int j = j0 + u * blockDim.x;
      if (j0 == (int)threadIdx.x) keep[u] = acc[u];
      if (j < p.H) {
        rb[j] = acc[u];
        ss += acc[u] * acc[u];
      }
    }
  }
  if (p.xnorm) {
    ss = block_sum(ss, red);
    const float inv = rsqrtf(ss / (float)p.H + p.eps);
    uint16_t* xn = p.xnorm + (size_t)b * p.H;
#pragma unroll
    for (int u = 0; u < kCombineU; ++u) {
      const int j = threadIdx.x + u * blockDim.x;
      if (j < p.H) xn[j] = f32_to_bf16_bits(keep[u] * inv);
    }
    for (int j = threadIdx.x + stride; j < p.H; j += blockDim.x) xn[j] = f32_to_bf16_bits(rb[j] * inv);
  }
}

// moe_rmsnorm: grid B, one token per CTA. xn = bf16(r * rsqrt(mean(r^2) +
// eps) * weight) with unit weight when none is given (the RMS norm kernel of
// the Flash-MoE page, "Metal Compute Shaders"). H a multiple of 8; r is read
// twice (the second time from L1/L2).
__global__ void __launch_bounds__(kCombineThreads) k_rmsnorm(const float* r, const uint16_t* weight, int H, float eps,
                                                             uint16_t* out) {
  __shared__ float red[32];
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, n4 = H / 4;
  const float4* rb = reinterpret_cast<const float4*>(r + (size_t)b * H);
  float ss = 0.f;
  for (int j = threadIdx.x; j < n4; j += blockDim.x) {
    const float4 v = rb[j];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)H + eps);
  uint2* ob = reinterpret_cast<uint2*>(out + (size_t)b * H);
  for (int j = threadIdx.x; j < n4; j += blockDim.x) {
    const float4 v = rb[j];
    float f[4] = {v.x * inv, v.y * inv, v.z * inv, v.w * inv};
    if (weight) {
      const uint2 wv = reinterpret_cast<const uint2*>(weight)[j];
      f[0] *= bf16_bits_to_f32(wv.x & 0xFFFFu);
      f[1] *= bf16_bits_to_f32(wv.x >> 16);
      f[2] *= bf16_bits_to_f32(wv.y & 0xFFFFu);
      f[3] *= bf16_bits_to_f32(wv.y >> 16);
    }
    ob[j] = make_uint2((uint32_t)f32_to_bf16_bits(f[0]) | ((uint32_t)f32_to_bf16_bits(f[1]) << 16),
                       (uint32_t)f32_to_bf16_bits(f[2]) | ((uint32_t)f32_to_bf16_bits(f[3]) << 16));
  }
}

}  // namespace moeq
