// common.cuh -- device helpers shared by the libmoeq kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moeq.h"

namespace moeq {

// Workspace control block: the first 256 bytes of every workspace.
struct WsCtrl {
  int error;                // first device-side moe_status (0 = none)
  unsigned router_ticket[16]; // last-CTA tickets of the router kernel, one per 8-token tile (0 between calls)
  unsigned exit_count;      // CTAs that left the fused decode kernel (0 between calls)
  unsigned sync[8];         // arrival counters of the fused decode kernel (0 between calls)
  unsigned wait_us;         // budget of every bounded wait in microseconds (0: about one second)
  int withhold_cta;         // c + 1: CTA c of the fused kernel withholds its first logits arrival (0: none)
  unsigned pad[36];
};
static_assert(sizeof(WsCtrl) == 256, "control block is 256 bytes");

constexpr size_t kAlign = 256;
__host__ __device__ inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }

__device__ __forceinline__ void set_error(WsCtrl* c, int code) {
  if (c) atomicCAS(&c->error, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// Round-to-nearest-even fp32 -> bf16 bits (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Geometry of one expert record (bytes). Every matrix is stored as tiles of
// 16 rows laid out for the int8 tensor-core dot (mma m16n8k32 fragments):
// tile T holds, for each group of G inputs, one block of
//   codes  32 lanes x (G/32 k-steps) x W bytes (W = 8 at 4 bits, 4 at 2 bits;
//          3 bits: a 2-bit plane of 4 bytes per lane and k-step, then a
//          1-bit plane of 2 bytes per lane and k-step)
//   table  8 x [(scale, bias) of local row g, (scale, bias) of local row g+8]
// Gate/up tile T (at T*U, I/8 tiles of H inputs) holds gate rows 8T..8T+7 as
// local rows 0..7 and up rows 8T..8T+7 as local rows 8..15; down tile T (at
// down_off + T*D, H/16 tiles of I inputs) holds rows 16T..16T+15.
constexpr int kTileRows = 16;
struct RecGeom {
  uint32_t blk;               // block bytes (one group of one tile)
  uint32_t ng_h, U;           // gate/up: groups per tile, tile bytes
  uint32_t ng_i, D;           // down: groups per tile, tile bytes
  unsigned long long down_off;
};
__host__ __device__ inline uint32_t tile_block_bytes(int bits, int group) {
  return (uint32_t)(2 * group * bits + 64);  // 16 rows x group codes of `bits` bits, then the tables
}
__host__ __device__ inline RecGeom rec_geom(int H, int I, int bits, int group) {
  RecGeom g;
  g.blk = tile_block_bytes(bits, group);
  g.ng_h = (uint32_t)(H / group);
  g.U = g.ng_h * g.blk;
  g.ng_i = (uint32_t)(I / group);
  g.D = g.ng_i * g.blk;
  g.down_off = (unsigned long long)(I / 8) * g.U;
  return g;
}

// Programmatic dependent launch (PTX griddepcontrol; no-ops when the launch
// did not ask for it). A kernel of the per-call chain lets the next one launch
// as soon as it starts (pdl_trigger first); the next one does only work that
// reads constant weights before pdl_wait, which returns once this grid has
// completed and its writes are visible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Streaming 16-byte load of weights that are read once: bypass L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream4(const void* p) {
  uint32_t v;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// Block-wide sum for blockDim.x a multiple of 32 (<= 1024); `red` holds 32 floats.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
  return warp_sum(t);
}

__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.f;
  return warp_max(t);
}

// 2^e as fp32 for e in [-126, 127].
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Power-of-two exponent that maps amax into [2^14, 2^15): values scaled by
// 2^e fit fp16 (max 65504) with headroom for the products of the dequant
// dot. Clamped so that 2^e and 2^-e are normal fp32 numbers.
__device__ __forceinline__ int fp16_scale_exp(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 0;
  int e = 15 - (((int)((__float_as_uint(amax) >> 23) & 0xFF)) - 126);
  return max(-120, min(120, e));
}

}  // namespace moeq

// ---- mbarriers, bulk async copies, bounded waits (sm_90+/sm_100a) ---------
namespace moeq {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p;\n\t mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bulk copy global -> this CTA's shared memory; completion counted in bytes
// on `bar`. Addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Bulk prefetch of global memory into L2 (no shared memory, no completion).
// Address 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide arrival: a release-ordered reduction (no returned value, so the
// arriving thread does not wait for the round trip). Writes of the whole CTA
// that were ordered before it by a CTA barrier become visible first.
__device__ __forceinline__ void arrive_release_gpu(unsigned* counter) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
}

// Default budget of every spin in the library: ~1 s of SM clock cycles.
constexpr long long kWaitBudgetCycles = 2000000000LL;

// The budget a kernel's waits use: the workspace's wait_us (a testing hook,
// about 2000 cycles per microsecond) or the default. Read once per kernel.
__device__ __forceinline__ long long wait_budget(const WsCtrl* c) {
  const unsigned us = c ? *reinterpret_cast<const volatile unsigned*>(&c->wait_us) : 0u;
  return us ? (long long)us * 2000LL : kWaitBudgetCycles;
}

// Bounded wait for an mbarrier phase; false after `budget` cycles or when
// `abort` is set. Waiting warps back off with __nanosleep so that they leave
// the issue slots to the warps that have work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort, long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(64);
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
}

__device__ __forceinline__ unsigned ld_relaxed_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *counter >= target (gpu-scope acquire). The poll reads
// relaxed; once the target is seen, one acquire read of the counter (the
// counts only grow) orders the caller's later reads after the arrivals.
__device__ __forceinline__ bool counter_wait(const unsigned* counter, unsigned target, const volatile int* abort,
                                             long long budget) {
  if (ld_acquire_gpu(counter) >= target) return true;
  const long long t0 = clock64();
  while (ld_relaxed_gpu(counter) < target) {
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
    __nanosleep(32);
  }
  (void)ld_acquire_gpu(counter);
  return true;
}

// Named barriers among a subset of the CTA's warps.
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace moeq
