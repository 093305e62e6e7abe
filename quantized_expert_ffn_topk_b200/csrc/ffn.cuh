// ffn.cuh -- moe_expert_ffn_q for one token: gate/up dequant mat-vecs with
// fused SwiGLU, then the down dequant mat-vec, for the K routed experts and
// the shared expert (the per-call path; the arithmetic of a tile is in
// tiledot.cuh; the steps are the Flash-MoE page's expert FFN, "Metal Compute
// Shaders").
//
// One CTA per SM. A CTA takes a contiguous share of the layer's tiles (split
// over all selected experts at once) and bulk-copies all of them into shared
// memory up front, each tile completing on its own mbarrier; while the copies
// are in flight it stages the input image, and its warps then take
// quarter-tile pieces as the tiles land. A share that does not fit shared
// memory is worked in rounds of as many tiles as fit.
#pragma once

#include "common.cuh"
#include "tiledot.cuh"

namespace moeq {

constexpr int kFfnWarps = 16;
// Pieces of a tile (each a contiguous part of its groups, one warp each): a
// CTA's share of 4 or 5 gate/up tiles in 3 pieces is one wave of the 16 warps
// (in 4, five tiles took two); down jobs stay in 4 (5 or 8 measured no faster)
#ifndef MOEQ_FFN_PIECES_GU
#define MOEQ_FFN_PIECES_GU 3
#endif
#ifndef MOEQ_FFN_PIECES_DN
#define MOEQ_FFN_PIECES_DN 4
#endif
constexpr int kFfnPiecesGu = MOEQ_FFN_PIECES_GU;
constexpr int kFfnPiecesDn = MOEQ_FFN_PIECES_DN;
constexpr int kFfnMaxBuf = 32;    // tile buffers (mbarriers) per CTA

struct FfnParams {
  const uint8_t* experts;    // E routed records
  const uint8_t* shared;     // shared record
  size_t rec_r;              // routed record bytes
  RecGeom geo_r, geo_s;      // record geometry, routed and shared
  const uint16_t* x;         // [B, H] bf16
  const int32_t* idx;        // [B, K]
  float* h;                  // [B, K+1, I] (workspace)
  float* y;                  // [B, K+1, H]
  WsCtrl* ctrl;
  int H, I, E, K, G, bits_r, bits_s, B;
  // shared-memory plans of the one-token kernels (byte offsets)
  int gu_nbuf, gu_gs, gu_part, gu_tiles, gu_stride;
  int dn_nbuf, dn_img_stride, dn_img_gs, dn_part, dn_tiles, dn_stride;
  int dn_ctas;  // CTAs of the down kernel
  // 1: the dots run on the CUDA cores in fp32 (tile_dot_fma) on fp32 copies
  // of the inputs at gu_xf / (image) + dn_img_xf, for comparison with the
  // tensor-core dot (0, the default)
  int dot_fma, gu_xf, dn_img_xf;
};

// Groups [lo, hi) of piece q of NP of a tile with ng groups.
template <int NP>
__host__ __device__ inline int piece_lo(int q, int ng) { return q * ng / NP; }

// Record of slot k of the token (routed expert idx[k], or the shared expert
// for k == K); null for an invalid expert index.
__device__ __forceinline__ const uint8_t* ffn_slot_rec(const FfnParams& p, int k) {
  if (k == p.K) return p.shared;
  const int e = p.idx[k];
  return (e >= 0 && e < p.E) ? p.experts + (size_t)e * p.rec_r : nullptr;
}

// Issue the bulk copies of tiles [u0, u0 + nt) of the CTA's share (lane j
// copies tile u0 + j into buffer j; 0 bytes for an invalid expert). `src`
// gives a tile's record, offset and size; `take(u)` selects which tiles this
// call issues (the gate/up kernel: the shared expert's before pdl_wait, the
// routed ones after).
template <typename Src, typename Take>
__device__ __forceinline__ void ffn_issue(unsigned char* tiles, int stride, uint64_t* bar, int u0, int nt, Src src,
                                          Take take) {
  const int lane = threadIdx.x & 31;
  for (int j = lane; j < nt; j += 32) {
    if (!take(u0 + j)) continue;
    const unsigned char* from = nullptr;
    const uint32_t bytes = src(u0 + j, &from);
    mbar_arrive_expect_tx(&bar[j], bytes);
    if (bytes) bulk_g2s(tiles + (size_t)j * stride, from, bytes, &bar[j]);
  }
}

// Bounded wait for buffer j of the current round; on a timeout the CTA
// records MOE_ERR_TIMEOUT and stops.
__device__ __forceinline__ bool ffn_wait(uint64_t* bar, int j, int round, WsCtrl* ctrl, volatile int* abort,
                                         long long budget) {
  const bool ok = mbar_wait(&bar[j], (uint32_t)(round & 1), abort, budget);
  if (!ok && (threadIdx.x & 31) == 0) {
    if (!*abort) set_error(ctrl, MOE_ERR_TIMEOUT);
    *abort = 1;
  }
  return ok;
}

// Before the CTA leaves after a timeout: every copy it issued must have
// landed (bounded).
__device__ __forceinline__ void ffn_drain(uint64_t* bar, int nt, int round, long long budget) {
  if (threadIdx.x < nt) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar[threadIdx.x], (uint32_t)(round & 1)) && clock64() - t0 < budget) {
    }
  }
}

// Gate/up: tile u = (slot u / (I/8), tile u % (I/8)) holds gate rows 8T..8T+7
// and up rows 8T..8T+7; 8 threads per tile finish h = SiLU(gate) * up.
__global__ void __launch_bounds__(kFfnWarps * 32, 1) k_gate_up(const __grid_constant__ FfnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar[kFfnMaxBuf];
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const QImg X{reinterpret_cast<uint2*>(smem), reinterpret_cast<float2*>(smem + p.gu_gs)};
  float* part = reinterpret_cast<float*>(smem + p.gu_part);  // [buffer][piece][16]
  unsigned char* tiles = smem + p.gu_tiles;
  const int tps = p.I / 8, total = (p.K + 1) * tps;
  const int t_lo = (int)((long long)total * blockIdx.x / gridDim.x);
  const int t_hi = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
  if (tid == 0) {
    for (int j = 0; j < p.gu_nbuf; ++j) mbar_init(&bar[j], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto src = [&](int u, const unsigned char** from) -> uint32_t {
    const int k = u / tps, T = u % tps;
    const uint8_t* rec = ffn_slot_rec(p, k);
    if (!rec) return 0u;
    const RecGeom& g = k < p.K ? p.geo_r : p.geo_s;
    *from = rec + (size_t)T * g.U;
    return g.U;
  };
  auto is_shared = [&](int u) { return u / tps == p.K; };
  auto is_routed = [&](int u) { return u / tps != p.K; };
  auto any = [&](int) { return true; };
  // the shared expert's tiles do not depend on the previous kernel
  if (warp == 0 && t_lo < t_hi) ffn_issue(tiles, p.gu_stride, bar, t_lo, min(p.gu_nbuf, t_hi - t_lo), src, is_shared);
  pdl_wait();
  // the down kernel may start from here on: the router has completed, so it
  // can read the picks and issue all its tile copies at once
  pdl_trigger();
  const long long budget = wait_budget(p.ctrl);
  int round = 0, nt = 0;
  for (int r0 = t_lo; r0 < t_hi; r0 += p.gu_nbuf, ++round) {
    nt = min(p.gu_nbuf, t_hi - r0);
    if (warp == 0) {
      if (r0 == t_lo) ffn_issue(tiles, p.gu_stride, bar, r0, nt, src, is_routed);
      else ffn_issue(tiles, p.gu_stride, bar, r0, nt, src, any);
    }

    if (r0 == t_lo) {  // the input image, while the first round's tiles are in flight
      float* xf = reinterpret_cast<float*>(smem + p.gu_xf);
      qstage_vector(
          [&](int j0, float (&v)[16]) {
            load_bf16_16(p.x + j0, v);
            if (p.dot_fma)
#pragma unroll
              for (int q = 0; q < 4; ++q)
                reinterpret_cast<float4*>(xf + j0)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          },
          p.H, p.G, X, tid, blockDim.x);
      __syncthreads();
    }
    for (int pc = warp; pc < nt * kFfnPiecesGu; pc += kFfnWarps) {
      const int j = pc / kFfnPiecesGu, q = pc % kFfnPiecesGu, k = (r0 + j) / tps;
      const bool routed = k < p.K;
      float acc0 = 0.f, acc1 = 0.f;
      if (ffn_wait(bar, j, round, p.ctrl, &s_abort, budget) && ffn_slot_rec(p, k)) {
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int g0 = piece_lo<kFfnPiecesGu>(q, (int)g.ng_h), g1 = piece_lo<kFfnPiecesGu>(q + 1, (int)g.ng_h);
        const unsigned char* blk = tiles + (size_t)j * p.gu_stride + (size_t)g0 * g.blk;
        const float* xf = reinterpret_cast<const float*>(smem + p.gu_xf);
        with_fmt(routed ? p.bits_r : p.bits_s, p.G, [&]<int BITS, int KS>() {
          if (p.dot_fma) tile_dot_fma<BITS, KS>(blk, g1 - g0, g0, xf, X.gs, acc0, acc1);
          else tile_dot<BITS, KS>(blk, g1 - g0, g0, X, acc0, acc1);
        });
      }
      if ((lane & 3) == 0) {
        float* pp = part + ((size_t)j * kFfnPiecesGu + q) * kTileRows;
        pp[lane >> 2] = acc0;
        pp[(lane >> 2) + 8] = acc1;
      }
    }
    __syncthreads();
    for (int i = tid; i < nt * 8; i += blockDim.x) {
      const int j = i / 8, unit = i % 8, u = r0 + j, k = u / tps, T = u % tps;
      float gate = 0.f, up = 0.f;
#pragma unroll
      for (int q = 0; q < kFfnPiecesGu; ++q) {
        gate += part[((size_t)j * kFfnPiecesGu + q) * kTileRows + unit];
        up += part[((size_t)j * kFfnPiecesGu + q) * kTileRows + 8 + unit];
      }
      const bool ok = ffn_slot_rec(p, k) != nullptr;
      if (!ok && unit == 0) set_error(p.ctrl, MOE_ERR_INDEX);
      p.h[(size_t)k * p.I + 8 * T + unit] = ok ? silu_f(gate) * up : 0.f;
    }
    __syncthreads();  // buffers and partials free for the next round
    if (s_abort) break;
  }
  if (s_abort) ffn_drain(bar, nt, round, budget);
}

// Down: job u = (slot u / (H/16), down tile u % (H/16)); 16 threads per job
// sum its pieces into y.
__global__ void __launch_bounds__(kFfnWarps * 32, 1) k_down(const __grid_constant__ FfnParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar[kFfnMaxBuf];
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* part = reinterpret_cast<float*>(smem + p.dn_part);  // [buffer][piece][16]
  unsigned char* tiles = smem + p.dn_tiles;
  const int tpd = p.H / kTileRows, total = (p.K + 1) * tpd;
  const int t_lo = (int)((long long)total * blockIdx.x / gridDim.x);
  const int t_hi = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
  auto img = [&](int k) {
    return QImg{reinterpret_cast<uint2*>(smem + (size_t)k * p.dn_img_stride),
                reinterpret_cast<float2*>(smem + (size_t)k * p.dn_img_stride + p.dn_img_gs)};
  };
  if (tid == 0) {
    for (int j = 0; j < p.dn_nbuf; ++j) mbar_init(&bar[j], 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  auto src = [&](int u, const unsigned char** from) -> uint32_t {
    const int k = u / tpd, T = u % tpd;
    const uint8_t* rec = ffn_slot_rec(p, k);
    if (!rec) return 0u;
    const RecGeom& g = k < p.K ? p.geo_r : p.geo_s;
    *from = rec + g.down_off + (size_t)T * g.D;
    return g.D;
  };
  auto any = [&](int) { return true; };
  // the tiles depend only on the weights and the picks: the gate/up kernel
  // lets this kernel start only after the router has completed, so the
  // first round's copies go out before the wait for the gate/up kernel's h
  if (warp == 0 && t_lo < t_hi) ffn_issue(tiles, p.dn_stride, bar, t_lo, min(p.dn_nbuf, t_hi - t_lo), src, any);
  pdl_wait();
  const long long budget = wait_budget(p.ctrl);
  int round = 0, nt = 0;
  for (int r0 = t_lo; r0 < t_hi; r0 += p.dn_nbuf, ++round) {
    nt = min(p.dn_nbuf, t_hi - r0);
    if (warp == 0 && r0 != t_lo) ffn_issue(tiles, p.dn_stride, bar, r0, nt, src, any);
    if (r0 == t_lo) {  // images of the slots this CTA's jobs touch
      for (int k = t_lo / tpd; k <= (t_hi - 1) / tpd; ++k) {
        const float* hk = p.h + (size_t)k * p.I;
        float* hf = reinterpret_cast<float*>(smem + (size_t)k * p.dn_img_stride + p.dn_img_xf);
        qstage_vector(
            [&](int j0, float (&v)[16]) {
              load_f32_16_cg(hk + j0, v);
              if (p.dot_fma)
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  reinterpret_cast<float4*>(hf + j0)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            },
            p.I, p.G, img(k), tid, blockDim.x);
      }
      __syncthreads();
    }
    for (int pc = warp; pc < nt * kFfnPiecesDn; pc += kFfnWarps) {
      const int j = pc / kFfnPiecesDn, q = pc % kFfnPiecesDn, k = (r0 + j) / tpd;
      const bool routed = k < p.K;
      float acc0 = 0.f, acc1 = 0.f;
      if (ffn_wait(bar, j, round, p.ctrl, &s_abort, budget) && ffn_slot_rec(p, k)) {
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int g0 = piece_lo<kFfnPiecesDn>(q, (int)g.ng_i), g1 = piece_lo<kFfnPiecesDn>(q + 1, (int)g.ng_i);
        const unsigned char* blk = tiles + (size_t)j * p.dn_stride + (size_t)g0 * g.blk;
        const QImg Hk = img(k);
        const float* hf = reinterpret_cast<const float*>(smem + (size_t)k * p.dn_img_stride + p.dn_img_xf);
        with_fmt(routed ? p.bits_r : p.bits_s, p.G, [&]<int BITS, int KS>() {
          if (p.dot_fma) tile_dot_fma<BITS, KS>(blk, g1 - g0, g0, hf, Hk.gs, acc0, acc1);
          else tile_dot<BITS, KS>(blk, g1 - g0, g0, Hk, acc0, acc1);
        });
      }
      if ((lane & 3) == 0) {
        float* pp = part + ((size_t)j * kFfnPiecesDn + q) * kTileRows;
        pp[lane >> 2] = acc0;
        pp[(lane >> 2) + 8] = acc1;
      }
    }
    __syncthreads();
    for (int i = tid; i < nt * kTileRows; i += blockDim.x) {
      const int j = i / kTileRows, rho = i % kTileRows, u = r0 + j, k = u / tpd, T = u % tpd;
      float y = 0.f;
#pragma unroll
      for (int q = 0; q < kFfnPiecesDn; ++q) y += part[((size_t)j * kFfnPiecesDn + q) * kTileRows + rho];
      p.y[(size_t)k * p.H + (size_t)T * kTileRows + rho] = y;
    }
    __syncthreads();
    if (s_abort) break;
  }
  if (s_abort) ffn_drain(bar, nt, round, budget);
}

}  // namespace moeq
