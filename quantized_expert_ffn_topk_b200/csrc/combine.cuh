// combine.cuh -- moe_combine_residual: weighted combine of the routed experts
// with the shared expert and the residual, optional shared-expert sigmoid
// gate, optional RMSNorm'd bf16 copy for the next layer (Flash-MoE page,
// sections "Metal Compute Shaders" and "Deferred GPU Expert Compute").
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace moeq {

constexpr int kCombineThreads = 512;
constexpr int kCombineCluster = 8;  // CTAs per token (a thread block cluster)

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

// Cluster shared-memory helpers: the address of the same variable in CTA
// `rank` of the cluster, a 4-byte store into it that completes `bytes` on
// that CTA's mbarrier, and a bounded wait on a local mbarrier phase whose
// data came from the cluster's CTAs.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_async_f32(uint32_t dst, float v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(dst),
               "r"(__float_as_uint(v)), "r"(bar)
               : "memory");
}
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, long long budget) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p;\n\t mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t selp.u32 %0, 1, "
        "0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > budget) return false;
  }
}

// grid: B clusters of kCombineCluster CTAs, one cluster per token; CTA rank
// q of a cluster owns elements [q*per, (q+1)*per) of its token (per =
// ceil(H / kCombineCluster)), one or a few per thread. The RMSNorm'd copy
// needs the token's whole sum of squares: each CTA reduces its part and
// stores it into every cluster peer's shared memory (st.async, counted on
// the peer's mbarrier), then adds the parts in rank order once its own
// barrier has them all. The only cluster barrier comes first (the peers'
// mbarriers armed, nothing stored yet), so no fence waits on the global
// stores of r; a CTA leaves only after every peer's part has landed in it.
// The first element of each thread has its inputs loaded before the gate's
// reduction. A part that never lands (after about a second) leaves the
// CTA's share of the bf16 copy NaN.
__global__ void __cluster_dims__(kCombineCluster, 1, 1) __launch_bounds__(kCombineThreads)
    k_combine(CombineParams p) {
  __shared__ float red[32];
  __shared__ float s_parts[kCombineCluster];
  __shared__ __align__(8) uint64_t s_bar;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int b = blockIdx.x / kCombineCluster, q = (int)cluster.block_rank();
  if (p.xnorm) {
    if (threadIdx.x == 0) {
      mbar_init(&s_bar, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(&s_bar, kCombineCluster * (uint32_t)sizeof(float));
    }
    cluster.sync();  // every peer's barrier is armed before any part is sent
  }
  pdl_trigger();
  pdl_wait();
  const uint16_t* xb = p.x + (size_t)b * p.H;
  const float* yb = p.y + (size_t)b * (p.K + 1) * p.H;
  float* rb = p.resid_out + (size_t)b * p.H;
  const int per = (p.H + kCombineCluster - 1) / kCombineCluster;
  const int j0 = q * per, j1 = min(p.H, j0 + per);
  const int ja = j0 + (int)threadIdx.x;
  float ra = 0.f, ya[MOEQ_MAX_K + 1];
#pragma unroll
  for (int k = 0; k <= MOEQ_MAX_K; ++k) ya[k] = 0.f;
  if (ja < j1) {
    ra = p.resid_in ? p.resid_in[(size_t)b * p.H + ja] : bf16_bits_to_f32(xb[ja]);
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_K; ++k)
      if (k <= p.K) ya[k] = yb[(size_t)k * p.H + ja];
  }
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
  float ss = 0.f, keep = 0.f;
  if (ja < j1) {
    float acc = ra;
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_K; ++k)
      if (k <= p.K) acc += wk[k] * ya[k];
    keep = acc;
    rb[ja] = acc;
    ss += acc * acc;
  }
  for (int j = ja + (int)blockDim.x; j < j1; j += blockDim.x) {
    float acc = p.resid_in ? p.resid_in[(size_t)b * p.H + j] : bf16_bits_to_f32(xb[j]);
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_K; ++k)
      if (k <= p.K) acc += wk[k] * yb[(size_t)k * p.H + j];
    rb[j] = acc;
    ss += acc * acc;
  }
  if (p.xnorm) {
    ss = block_sum(ss, red);
    if (threadIdx.x < kCombineCluster)  // thread r sends this CTA's part to rank r
      st_async_f32(cluster_addr(&s_parts[q], threadIdx.x), ss, cluster_addr(&s_bar, threadIdx.x));
    const bool ok = mbar_wait_cluster(&s_bar, 0, kWaitBudgetCycles);
    float tot = 0.f;
#pragma unroll
    for (int r = 0; r < kCombineCluster; ++r) tot += s_parts[r];
    const float inv = ok ? rsqrtf(tot / (float)p.H + p.eps) : __int_as_float(0x7FC00000);
    uint16_t* xn = p.xnorm + (size_t)b * p.H;
    for (int j = ja; j < j1; j += blockDim.x) xn[j] = f32_to_bf16_bits((j == ja ? keep : rb[j]) * inv);
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
