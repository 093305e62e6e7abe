// ffn.cuh -- moe_expert_ffn_q: gate/up dequant mat-vecs with fused SwiGLU,
// then the down dequant mat-vec, for the K routed experts and the shared
// expert of each token (the per-call path; the arithmetic of a tile is in
// tiledot.cuh). Weights stream from global memory straight into registers.
#pragma once

#include "common.cuh"
#include "tiledot.cuh"

namespace moeq {

constexpr int kFfnWarps = 8;
constexpr int kFfnPieces = 4;   // warps per tile: each takes a quarter of the tile's groups
constexpr int kFfnPrefetch = 4; // blocks in flight per warp

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
  int tiles_per_cta_gu;      // gate/up tiles (slot-major, (K+1)*I/8 per token) per CTA
  int jobs_per_cta_dn;       // down jobs (slot, tile), (K+1)*H/16 per token, per CTA
};

// Groups [lo, hi) of piece q of a tile with ng groups.
__host__ __device__ inline int piece_lo(int q, int ng) { return q * ng / kFfnPieces; }

// Shared memory of the gate/up kernel: x's image and the per-round partials.
__host__ __device__ inline int gu_smem_bytes(int H, int G) {
  return (int)(align_up(qimg_plane_bytes(H), 16) + align_up(qimg_gs_bytes(H, G), 16)) +
         (kFfnWarps / kFfnPieces) * kFfnPieces * kTileRows * 4;
}

// Persistent over tiles: grid (ctas, B); CTA c takes tiles [c*tpc, (c+1)*tpc)
// of token blockIdx.y, tile u = (slot u / (I/8), tile u % (I/8)). Each round
// two tiles are split into four pieces, one per warp; the partial sums meet
// in shared memory and 16 threads finish h for the two tiles' 16 units.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_gate_up(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  QImg X{reinterpret_cast<uint2*>(smem),
         reinterpret_cast<float2*>(smem + align_up(qimg_plane_bytes(p.H), 16))};
  float* part = reinterpret_cast<float*>(smem + align_up(qimg_plane_bytes(p.H), 16) +
                                         align_up(qimg_gs_bytes(p.H, p.G), 16));  // [2][4][16]
  pdl_wait();
  const uint16_t* xb = p.x + (size_t)b * p.H;
  qstage_vector([&](int j0, float (&v)[16]) { load_bf16_16(xb + j0, v); }, p.H, p.G, X, threadIdx.x, blockDim.x);
  __syncthreads();

  const int tiles_per_slot = p.I / 8;
  const int total = (p.K + 1) * tiles_per_slot;
  const int t_begin = blockIdx.x * p.tiles_per_cta_gu;
  const int t_end = min(total, t_begin + p.tiles_per_cta_gu);
  constexpr int kPerRound = kFfnWarps / kFfnPieces;
  for (int t0 = t_begin; t0 < t_end; t0 += kPerRound) {
    const int u = t0 + warp / kFfnPieces, q = warp % kFfnPieces;
    float acc0 = 0.f, acc1 = 0.f;
    bool bad = false;
    if (u < t_end) {
      const int k = u / tiles_per_slot, T = u % tiles_per_slot;
      const bool routed = k < p.K;
      const int e = routed ? p.idx[(size_t)b * p.K + k] : 0;
      bad = routed && (e < 0 || e >= p.E);
      if (!bad) {
        const uint8_t* rec = routed ? p.experts + (size_t)e * p.rec_r : p.shared;
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int g0 = piece_lo(q, g.ng_h), g1 = piece_lo(q + 1, g.ng_h);
        const unsigned char* blk = rec + (size_t)T * g.U + (size_t)g0 * g.blk;
        with_fmt(routed ? p.bits_r : p.bits_s, p.G, [&]<int BITS, int KS>() {
          tile_dot_global<BITS, KS, kFfnPrefetch>(blk, g1 - g0, g0, X, acc0, acc1);
        });
      } else if (lane == 0 && q == 0) {
        set_error(p.ctrl, MOE_ERR_INDEX);
      }
    }
    if ((lane & 3) == 0) {
      float* pp = part + ((warp / kFfnPieces) * kFfnPieces + q) * kTileRows;
      pp[lane >> 2] = bad ? 0.f : acc0;
      pp[(lane >> 2) + 8] = bad ? 0.f : acc1;
    }
    __syncthreads();
    if (threadIdx.x < kPerRound * 8) {
      const int r = threadIdx.x / 8, unit = threadIdx.x % 8, tu = t0 + r;
      if (tu < t_end) {
        float gate = 0.f, up = 0.f;
#pragma unroll
        for (int qq = 0; qq < kFfnPieces; ++qq) {
          gate += part[(r * kFfnPieces + qq) * kTileRows + unit];
          up += part[(r * kFfnPieces + qq) * kTileRows + 8 + unit];
        }
        const int k = tu / tiles_per_slot, T = tu % tiles_per_slot;
        p.h[((size_t)b * (p.K + 1) + k) * p.I + 8 * T + unit] = silu_f(gate) * up;
      }
    }
    __syncthreads();
  }
  pdl_trigger();
}

// Shared memory of the down kernel: one image of h per slot, then partials.
struct DnSmem {
  int planes_stride, gs_off, gs_stride, part, bytes;
};
__host__ __device__ inline DnSmem dn_smem_plan(int I, int K, int G) {
  DnSmem s{};
  s.planes_stride = (int)align_up(qimg_plane_bytes(I), 16);
  s.gs_off = s.planes_stride * (K + 1);
  s.gs_stride = (int)align_up(qimg_gs_bytes(I, G), 16);
  s.part = s.gs_off + s.gs_stride * (K + 1);
  s.bytes = s.part + (kFfnWarps / kFfnPieces) * kFfnPieces * kTileRows * 4;
  return s;
}

__device__ __forceinline__ QImg dn_img(unsigned char* smem, const DnSmem& sp, int k) {
  return QImg{reinterpret_cast<uint2*>(smem + (size_t)k * sp.planes_stride),
              reinterpret_cast<float2*>(smem + sp.gs_off + (size_t)k * sp.gs_stride)};
}

// Persistent over jobs: grid (ctas, B); job u = (slot u / (H/16), down tile
// u % (H/16)). Two jobs per round, four pieces each; 32 threads sum the
// pieces into y.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_down(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DnSmem sp = dn_smem_plan(p.I, p.K, p.G);
  float* part = reinterpret_cast<float*>(smem + sp.part);
  pdl_wait();
  const float* hb = p.h + (size_t)b * (p.K + 1) * p.I;
  for (int k = 0; k <= p.K; ++k) {
    const float* hk = hb + (size_t)k * p.I;
    qstage_vector([&](int j0, float (&v)[16]) { load_f32_16_cg(hk + j0, v); }, p.I, p.G, dn_img(smem, sp, k),
                  threadIdx.x, blockDim.x);
  }
  __syncthreads();

  const int tiles_per_slot = p.H / kTileRows;
  const int total = (p.K + 1) * tiles_per_slot;
  const int j_begin = blockIdx.x * p.jobs_per_cta_dn;
  const int j_end = min(total, j_begin + p.jobs_per_cta_dn);
  constexpr int kPerRound = kFfnWarps / kFfnPieces;
  for (int j0 = j_begin; j0 < j_end; j0 += kPerRound) {
    const int u = j0 + warp / kFfnPieces, q = warp % kFfnPieces;
    float acc0 = 0.f, acc1 = 0.f;
    if (u < j_end) {
      const int k = u / tiles_per_slot, T = u % tiles_per_slot;
      const bool routed = k < p.K;
      const int e = routed ? p.idx[(size_t)b * p.K + k] : 0;
      if (!routed || (e >= 0 && e < p.E)) {
        const uint8_t* rec = routed ? p.experts + (size_t)e * p.rec_r : p.shared;
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int g0 = piece_lo(q, g.ng_i), g1 = piece_lo(q + 1, g.ng_i);
        const unsigned char* blk = rec + g.down_off + (size_t)T * g.D + (size_t)g0 * g.blk;
        const QImg Xk = dn_img(smem, sp, k);
        with_fmt(routed ? p.bits_r : p.bits_s, p.G, [&]<int BITS, int KS>() {
          tile_dot_global<BITS, KS, kFfnPrefetch>(blk, g1 - g0, g0, Xk, acc0, acc1);
        });
      }
    }
    if ((lane & 3) == 0) {
      float* pp = part + ((warp / kFfnPieces) * kFfnPieces + q) * kTileRows;
      pp[lane >> 2] = acc0;
      pp[(lane >> 2) + 8] = acc1;
    }
    __syncthreads();
    if (threadIdx.x < kPerRound * kTileRows) {
      const int r = threadIdx.x / kTileRows, rho = threadIdx.x % kTileRows, ju = j0 + r;
      if (ju < j_end) {
        float y = 0.f;
#pragma unroll
        for (int qq = 0; qq < kFfnPieces; ++qq) y += part[(r * kFfnPieces + qq) * kTileRows + rho];
        const int k = ju / tiles_per_slot, T = ju % tiles_per_slot;
        p.y[((size_t)b * (p.K + 1) + k) * p.H + (size_t)T * kTileRows + rho] = y;
      }
    }
    __syncthreads();
  }
  pdl_trigger();
}

}  // namespace moeq
