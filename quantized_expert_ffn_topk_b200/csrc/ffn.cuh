// ffn.cuh -- moe_expert_ffn_q: gate/up dequant mat-vecs with fused SwiGLU,
// then the down dequant mat-vec, for the K routed experts and the shared
// expert of each token (the per-call path; the arithmetic of a row is in
// dqdot.cuh).
#pragma once

#include "common.cuh"
#include "dqdot.cuh"

namespace moeq {

constexpr int kFfnWarps = 8;

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
  int units_per_cta_gu;      // gate/up units (slot, row) per CTA
  int units_per_cta_dn;      // down units per CTA
};

// NR rows sharing one input image, dotted by one warp. Lane l takes chunks
// l, l+32, ...; the loads of U chunk columns of all NR rows are issued before
// any arithmetic. Returns (in lane l) row l >> (5 - log2 NR)'s dot product,
// still multiplied by the image's 2^e.
template <int BITS, int NR, int U>
__device__ __forceinline__ float rows_dot(const uint8_t* const* codes, const uint32_t* const* sbrow, int ncols, int G,
                                          const ImgRef& R) {
  const int lane = threadIdx.x & 31;
  const int nchunk = ncols * BITS / 128;
  const bool two = (BITS == 2) && (G == 32);  // 2-bit codes, group 32: a chunk spans two groups
  float part[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) part[r] = 0.f;
  for (int c0 = lane; c0 < nchunk; c0 += 32 * U) {
    uint4 q[U][NR];
    uint32_t s0[U][NR], s1[U][NR];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        const int g = chunk_group<BITS>(c, G, two);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          q[u][r] = ld_stream16(codes[r] + (size_t)c * 16);
          s0[u][r] = ld_stream4(sbrow[r] + g);
          s1[u][r] = two ? ld_stream4(sbrow[r] + g + 1) : 0u;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c < nchunk) {
        const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, R);
#pragma unroll
        for (int r = 0; r < NR; ++r) part[r] += chunk_dot_x<BITS>(q[u][r], X, s0[u][r], s1[u][r], two);
      }
    }
  }
  return transpose_reduce<NR>(part);
}

// Shared-memory plan of the gate/up kernel: the image of x for each width in use.
struct GuSmem {
  int img4, tab4, inv4, img2, tab2, inv2, bytes;
};
__host__ __device__ inline GuSmem gu_smem_plan(int H, bool need4, bool need2) {
  GuSmem s{};
  size_t o = 0;
  auto take = [&](size_t b) {
    const size_t at = o;
    o += align_up(b, 16);
    return (int)at;
  };
  s.img4 = take(need4 ? img_bytes(H) : 0);
  s.tab4 = take(need4 ? tab_bytes(H, 4) : 0);
  s.inv4 = take(need4 ? inv_bytes(H, 4) : 0);
  s.img2 = take(need2 ? img_bytes(H) : 0);
  s.tab2 = take(need2 ? tab_bytes(H, 2) : 0);
  s.inv2 = take(need2 ? inv_bytes(H, 2) : 0);
  s.bytes = (int)o;
  return s;
}

// The CTA stages x straight from global memory, 16 inputs per thread.
template <int BITS>
__device__ __forceinline__ void stage_x_chunks(const uint16_t* xb, int H, ImgRef R) {
  stage_vector<BITS>([&](int j0, float (&v)[16]) { load_bf16_16(xb + j0, v); }, H, R, threadIdx.x, blockDim.x);
}

// Persistent over units: grid (ctas, B), CTA c takes units
// [c*upc, (c+1)*upc) of token blockIdx.y, unit u = (slot u / I, row u % I);
// a warp computes the gate row and the up row of one unit together.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_gate_up(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int b = blockIdx.y;
  const bool need4 = p.bits_r == 4 || p.bits_s == 4, need2 = p.bits_r == 2 || p.bits_s == 2;
  const GuSmem sp = gu_smem_plan(p.H, need4, need2);
  const ImgRef R4{reinterpret_cast<uint4*>(smem + sp.img4), reinterpret_cast<float4*>(smem + sp.tab4),
                  reinterpret_cast<float*>(smem + sp.inv4)};
  const ImgRef R2{reinterpret_cast<uint4*>(smem + sp.img2), reinterpret_cast<float4*>(smem + sp.tab2),
                  reinterpret_cast<float*>(smem + sp.inv2)};
  pdl_wait();
  const uint16_t* xb = p.x + (size_t)b * p.H;
  if (need4) stage_x_chunks<4>(xb, p.H, R4);
  if (need2) stage_x_chunks<2>(xb, p.H, R2);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total = (p.K + 1) * p.I;
  const int u_begin = blockIdx.x * p.units_per_cta_gu;
  const int u_end = min(total, u_begin + p.units_per_cta_gu);
  for (int u = u_begin + warp; u < u_end; u += kFfnWarps) {
    const int k = u / p.I, i = u % p.I;
    const bool routed = k < p.K;
    int e = routed ? p.idx[(size_t)b * p.K + k] : 0;
    float hval = 0.f;
    if (routed && (e < 0 || e >= p.E)) {
      if (lane == 0) set_error(p.ctrl, MOE_ERR_INDEX);
    } else {
      const uint8_t* rec = routed ? p.experts + (size_t)e * p.rec_r : p.shared;
      const RecGeom& g = routed ? p.geo_r : p.geo_s;
      const int bits = routed ? p.bits_r : p.bits_s;
      const uint8_t* unit = rec + (size_t)i * g.U;
      const uint8_t* codes[2] = {unit, unit + g.rowb_h};
      const uint32_t* sbr[2] = {reinterpret_cast<const uint32_t*>(unit + 2 * g.rowb_h),
                                reinterpret_cast<const uint32_t*>(unit + 2 * g.rowb_h + g.sbb_h)};
      const float v = bits == 4 ? rows_dot<4, 2, 4>(codes, sbr, p.H, p.G, R4) : rows_dot<2, 2, 2>(codes, sbr, p.H, p.G, R2);
      const float up = __shfl_sync(0xFFFFFFFFu, v, 16);  // lanes 16..31 hold the up row
      hval = silu_f(v) * up;
    }
    if (lane == 0) p.h[((size_t)b * (p.K + 1) + k) * p.I + i] = hval;
  }
  pdl_trigger();
}

// Shared-memory plan of the down kernel: one image of h per slot.
struct DnSmem {
  int img, tab, inv, img_stride, tab_stride, inv_stride, bytes;
};
__host__ __device__ inline DnSmem dn_smem_plan(int I, int K) {
  DnSmem s{};
  s.img_stride = (int)align_up(img_bytes(I), 16);
  s.tab_stride = (int)align_up(tab_bytes(I, 4), 16);  // 4-bit has the most chunks
  s.inv_stride = (int)align_up(inv_bytes(I, 4), 16);
  s.img = 0;
  s.tab = s.img_stride * (K + 1);
  s.inv = s.tab + s.tab_stride * (K + 1);
  s.bytes = s.inv + s.inv_stride * (K + 1);
  return s;
}

__device__ __forceinline__ ImgRef dn_img(unsigned char* smem, const DnSmem& sp, int k) {
  return ImgRef{reinterpret_cast<uint4*>(smem + sp.img + (size_t)k * sp.img_stride),
                reinterpret_cast<float4*>(smem + sp.tab + (size_t)k * sp.tab_stride),
                reinterpret_cast<float*>(smem + sp.inv + (size_t)k * sp.inv_stride)};
}

// Stage h (fp32, [K+1, I]) of one token: warp job j = (slot, 32 segments of
// 16 inputs), so that every warp stages one width at a time.
__device__ __forceinline__ void stage_h(const float* hb, int I, int K, int bits_r, int bits_s, unsigned char* smem,
                                        const DnSmem& sp, int tid, int nthr) {
  const int jobs_per_slot = (I / 16 + 31) / 32;
  const int lane = tid & 31;
  for (int j = tid >> 5; j < (K + 1) * jobs_per_slot; j += nthr >> 5) {
    const int k = j / jobs_per_slot, gi = j % jobs_per_slot;
    const float* hk = hb + (size_t)k * I;
    const ImgRef R = dn_img(smem, sp, k);
    auto get = [&](int j0, float (&v)[16]) { load_f32_16_cg(hk + j0, v); };
    if ((k < K ? bits_r : bits_s) == 4)
      stage_group<4>(get, I, R, gi, lane);
    else
      stage_group<2>(get, I, R, gi, lane);
  }
}

constexpr int kDownRows = 8;  // rows of one slot per warp unit

// Persistent over units: grid (ctas, B), unit u = (slot u / (H/8), block of
// 8 rows); a warp computes 8 rows of one slot at once.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_down(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DnSmem sp = dn_smem_plan(p.I, p.K);
  pdl_wait();
  stage_h(p.h + (size_t)b * (p.K + 1) * p.I, p.I, p.K, p.bits_r, p.bits_s, smem, sp, threadIdx.x, blockDim.x);
  __syncthreads();

  const int blocks_per_slot = p.H / kDownRows;
  const int total = (p.K + 1) * blocks_per_slot;
  const int u_begin = blockIdx.x * p.units_per_cta_dn;
  const int u_end = min(total, u_begin + p.units_per_cta_dn);
  for (int u = u_begin + warp; u < u_end; u += kFfnWarps) {
    const int k = u / blocks_per_slot, i0 = (u % blocks_per_slot) * kDownRows;
    const bool routed = k < p.K;
    const int e = routed ? p.idx[(size_t)b * p.K + k] : 0;
    float yval = 0.f;
    if (!(routed && (e < 0 || e >= p.E))) {
      const uint8_t* rec = routed ? p.experts + (size_t)e * p.rec_r : p.shared;
      const RecGeom& g = routed ? p.geo_r : p.geo_s;
      const int bits = routed ? p.bits_r : p.bits_s;
      const uint8_t* codes[kDownRows];
      const uint32_t* sbr[kDownRows];
#pragma unroll
      for (int r = 0; r < kDownRows; ++r) {
        const int row = i0 + r, rr = row % kRowsPerDownBlock;
        const uint8_t* blk = rec + g.down_off + (size_t)(row / kRowsPerDownBlock) * g.D;
        codes[r] = blk + (size_t)rr * g.rowb_i;
        sbr[r] = reinterpret_cast<const uint32_t*>(blk + kRowsPerDownBlock * g.rowb_i + (size_t)rr * g.sbb_i);
      }
      const ImgRef R = dn_img(smem, sp, k);
      yval = bits == 4 ? rows_dot<4, kDownRows, 1>(codes, sbr, p.I, p.G, R)
                       : rows_dot<2, kDownRows, 1>(codes, sbr, p.I, p.G, R);
    }
    if ((lane & 3) == 0) p.y[((size_t)b * (p.K + 1) + k) * p.H + i0 + (lane >> 2)] = yval;
  }
  pdl_trigger();
}

}  // namespace moeq
