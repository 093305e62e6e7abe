// tiledot.cuh -- the group-affine dequant dot product on the tensor cores.
//
// A row of a code matrix against an input vector x (w = q*scale + bias per
// group of G consecutive inputs) is
//   sum_j w_j x_j = sum_g [ scale_g * sum_{j in g} q_j x_j + bias_g * sum_{j in g} x_j ]
// the group-summed form of the Flash-MoE page's fma(q, scale*x, bias*x)
// (section "Kernel dequant toi uu FMA"): scale and bias are applied once per
// group, never per weight.
//
// The inner sums sum q_j x_j run on the tensor cores as exact integer
// arithmetic (mma.sync m16n8k32, u8 codes times s8 inputs, s32 accumulate):
//   - x is staged once per vector as a 16-bit fixed-point "image": within
//     group g every input becomes the integer v = rint(x * 2^F_g), with F_g the
//     largest exponent that keeps |v| <= 32639, split as v = 256*hi + lo with
//     hi, lo in [-128, 127]. hi feeds column 0 of the mma's B operand and lo
//     column 1, so one mma yields sum q*hi and sum q*lo for 16 rows and 32
//     inputs; 256*D_hi + D_lo is sum q*v exactly.
//   - codes come straight from the record's tile blocks, which hold each
//     lane's A fragments contiguously; 4-bit codes become u8 with one AND (low
//     nibbles) or a shift and an AND (high nibbles), 2-bit codes with a shift
//     and an AND per quarter.
//   - per group and row, acc += scale * (sum q*v) * 2^-F_g + bias * sum(x),
//     with sum(x) the exact fp32 sum of the group's inputs.
// The only rounding before the fp32 epilogue is that of x to 16 bits relative
// to its group's largest magnitude.
//
// Fragment layout (m16n8k32, lane = 4*gid + t): A register a0 holds row gid,
// k = 4t..4t+3; a1 row gid+8, the same k; a2 row gid, k = 16+4t..16+4t+3; a3
// row gid+8, k = 16+4t... B register b0 holds k = 4t..4t+3 of column gid, b1
// k = 16+4t... Accumulator c0/c1 are (row gid, columns 2t, 2t+1), c2/c3 (row
// gid+8, same columns). Within k-step m of a group the mma's k index maps to
// inputs: k = 4t + i <-> input 32m + 8t + 2i, and k = 16 + 4t + i <-> input
// 32m + 8t + 2i + 1; the packer and the image follow the same map.
#pragma once

#include "common.cuh"

namespace moeq {

// ---- the input image ------------------------------------------------------
//   planes  uint2 [n/32][8]: k-step m, column c (0: hi, 1: lo), lane t at
//           m*8 + 4c + t = (b0, b1), byte i of b0 = input 32m+8t+2i, of b1 =
//           input 32m+8t+2i+1
//   gs      float2 [n/G]: (2^-F_g, sum of the group's inputs)
struct QImg {
  uint2* planes;
  float2* gs;
};
__host__ __device__ inline size_t qimg_plane_bytes(int n) { return (size_t)n * 2; }
__host__ __device__ inline size_t qimg_gs_bytes(int n, int G) { return (size_t)(n / G) * 8; }

__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Stage segment s (inputs 16s..16s+15, values v) of a vector with groups of G
// (32, 64 or 128) inputs. G/16 adjacent lanes share a group; all 32 lanes of
// the warp call together, lanes without a segment with active = false (their
// values zero).
__device__ __forceinline__ void qstage_seg(const float (&v)[16], int s, int G, QImg Q, bool active) {
  const int gl = G >> 4;
  float amax = 0.f, sum = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    amax = fmaxf(amax, fabsf(v[j]));
    sum += v[j];
  }
  for (int o = 1; o < gl; o <<= 1) {
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  }
  // F: amax * 2^F <= 32639, as large as that allows (clamped to normal scales)
  const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
  int F = 14 - e;
  F = min(F, 126);
  if (amax * __uint_as_float((uint32_t)(F + 127) << 23) > 32639.f) F -= 1;
  F = max(F, -126);
  const float sc = __uint_as_float((uint32_t)(F + 127) << 23);
  int hi[16], lo[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int q = __float2int_rn(v[j] * sc);
    hi[j] = (q + 128) >> 8;
    lo[j] = q - (hi[j] << 8);
  }
  if (active) {
    const int m = s >> 1, p = s & 1;
    uint4* row = reinterpret_cast<uint4*>(Q.planes + (size_t)m * 8);
    row[p] = make_uint4(pack4_s8(hi[0], hi[2], hi[4], hi[6]), pack4_s8(hi[1], hi[3], hi[5], hi[7]),
                        pack4_s8(hi[8], hi[10], hi[12], hi[14]), pack4_s8(hi[9], hi[11], hi[13], hi[15]));
    row[2 + p] = make_uint4(pack4_s8(lo[0], lo[2], lo[4], lo[6]), pack4_s8(lo[1], lo[3], lo[5], lo[7]),
                            pack4_s8(lo[8], lo[10], lo[12], lo[14]), pack4_s8(lo[9], lo[11], lo[13], lo[15]));
    if ((s & (gl - 1)) == 0) Q.gs[s / gl] = make_float2(__uint_as_float((uint32_t)(127 - F) << 23), sum);
  }
}

// 16 bf16 inputs (global or shared memory, 16-byte aligned) -> fp32 values.
__device__ __forceinline__ void load_bf16_16(const uint16_t* src, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint4 w = reinterpret_cast<const uint4*>(src)[q];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(ww[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
  }
}

// 16 fp32 inputs written by an earlier kernel (read at L2).
__device__ __forceinline__ void load_f32_16_cg(const float* src, float (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 f = __ldcg(reinterpret_cast<const float4*>(src) + q);
    v[4 * q] = f.x;
    v[4 * q + 1] = f.y;
    v[4 * q + 2] = f.z;
    v[4 * q + 3] = f.w;
  }
}

// Stage a whole vector of n inputs (n a multiple of G) with nthr threads (a
// multiple of 32); get(j0, v) fills the 16 values starting at input j0.
template <typename Get>
__device__ __forceinline__ void qstage_vector(Get get, int n, int G, QImg Q, int tid, int nthr) {
  for (int s0 = tid - (tid & 31); s0 < n / 16; s0 += nthr) {
    const int s = s0 + (tid & 31);
    const bool active = s < n / 16;
    float v[16];
    if (active) {
      get(s * 16, v);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.f;
    }
    qstage_seg(v, s, G, Q, active);
  }
}

// ---- the tile dot ---------------------------------------------------------

// The mma has no side effect, so it is not volatile: the compiler may
// schedule it among the surrounding loads and the other groups' work.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint2 b, bool accumulate) {
  if (accumulate) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y));
  } else {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "r"(0));
  }
}

// Bytes of a block's code planes. 4 and 2 bits: one plane, LB bytes per lane
// (lane L at L*LB). 3 bits: the low 2 bits of every code in the 2-bit layout
// (4 bytes per lane and k-step, lane L at L*4*KS), then their third bits
// (2 bytes per lane and k-step, lane L at 128*KS + L*2*KS); in the third-bit
// word of k-steps 2p and 2p+1, bit 8i + 4*(ks & 1) + r is the third bit of
// byte i of A register r.
template <int BITS, int KS>
struct TileFmt {
  static_assert(BITS != 3 || KS % 2 == 0, "3-bit blocks need an even number of k-steps (group >= 64)");
  static constexpr int W = BITS == 4 ? 8 : 4;          // bytes per lane per k-step of the first plane
  static constexpr int LB = KS * W;                     // first-plane bytes per lane
  static constexpr int LH = BITS == 3 ? KS * 2 : 0;     // third-bit plane bytes per lane
  static constexpr int NW = (LB + LH) / 4;              // code words per lane
  static constexpr int CB = 32 * (LB + LH);             // code bytes per block
  static constexpr int BB = CB + 64;                    // block bytes
};

// A fragments of k-step ks from the lane's words w (NW of them).
template <int BITS, int KS>
__device__ __forceinline__ void extract_a(const uint32_t* w, int ks, uint32_t (&a)[4]) {
  if (BITS == 4) {
    const uint32_t w0 = w[2 * ks], w1 = w[2 * ks + 1];
    a[0] = w0 & 0x0F0F0F0Fu;
    a[1] = w1 & 0x0F0F0F0Fu;
    a[2] = (w0 >> 4) & 0x0F0F0F0Fu;
    a[3] = (w1 >> 4) & 0x0F0F0F0Fu;
  } else {
    const uint32_t w0 = w[ks];
    a[0] = w0 & 0x03030303u;
    a[1] = (w0 >> 2) & 0x03030303u;
    a[2] = (w0 >> 4) & 0x03030303u;
    a[3] = (w0 >> 6) & 0x03030303u;
    if (BITS == 3) {
      const uint32_t h = w[KS + (ks >> 1)] >> (4 * (ks & 1));
      a[0] |= (h & 0x01010101u) << 2;
      a[1] |= ((h >> 1) & 0x01010101u) << 2;
      a[2] |= ((h >> 2) & 0x01010101u) << 2;
      a[3] |= ((h >> 3) & 0x01010101u) << 2;
    }
  }
}

template <int NB>
__device__ __forceinline__ void load_words(const unsigned char* p, uint32_t* w) {
  if (NB >= 16) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 q = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = q.x;
      w[4 * i + 1] = q.y;
      w[4 * i + 2] = q.z;
      w[4 * i + 3] = q.w;
    }
  } else if (NB == 8) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    w[0] = q.x;
    w[1] = q.y;
  } else {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  }
}

// The lane's code words of one block (shared or global memory, plain loads).
template <int BITS, int KS>
__device__ __forceinline__ void load_lane_codes(const unsigned char* blk, int lane, uint32_t (&w)[TileFmt<BITS, KS>::NW]) {
  using F = TileFmt<BITS, KS>;
  load_words<F::LB>(blk + lane * F::LB, w);
  if (BITS == 3) load_words<F::LH>(blk + 32 * F::LB + lane * F::LH, w + F::LB / 4);
}

// One block (group g of a tile) from the lane's code words w and table pair
// sb against image X; adds into acc0 (local row gid) and acc1 (row gid+8).
template <int BITS, int KS>
__device__ __forceinline__ void block_acc(const uint32_t* w, uint2 sb, int g, const QImg& X, float& acc0,
                                          float& acc1) {
  const int lane = threadIdx.x & 31;
  const uint2* planes = X.planes + ((lane >> 2) & 1) * 4 + (lane & 3);
  int d[4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    uint32_t a[4];
    extract_a<BITS, KS>(w, ks, a);
    mma_u8s8(d, a, planes[(size_t)(g * KS + ks) * 8], ks > 0);
  }
  const float2 ms = X.gs[g];
  const float p0 = (float)(d[0] * 256 + d[1]) * ms.x;
  const float p1 = (float)(d[2] * 256 + d[3]) * ms.x;
  acc0 = fmaf(__uint_as_float(sb.x << 16), p0, acc0);
  acc0 = fmaf(__uint_as_float(sb.x & 0xFFFF0000u), ms.y, acc0);
  acc1 = fmaf(__uint_as_float(sb.y << 16), p1, acc1);
  acc1 = fmaf(__uint_as_float(sb.y & 0xFFFF0000u), ms.y, acc1);
}

// Groups of a tile dot whose loads and mma chains the compiler interleaves.
#ifndef MOEQ_TILE_UNROLL
#define MOEQ_TILE_UNROLL 2
#endif
constexpr int kTileUnroll = MOEQ_TILE_UNROLL;

// Blocks [0, nblk) of one tile in shared memory (at blk0, consecutive)
// against groups [g0, g0+nblk) of image X. Every lane of a row quad ends with
// the same values.
#ifdef MOEQ_TILE_NOINLINE
#define MOEQ_TILE_INLINE __noinline__
#else
#define MOEQ_TILE_INLINE __forceinline__
#endif
template <int BITS, int KS>
__device__ MOEQ_TILE_INLINE void tile_dot(const unsigned char* blk0, int nblk, int g0, const QImg& X, float& acc0,
                                          float& acc1) {
  using F = TileFmt<BITS, KS>;
  const int lane = threadIdx.x & 31;
#pragma unroll kTileUnroll
  for (int b = 0; b < nblk; ++b) {
    const unsigned char* blk = blk0 + (size_t)b * F::BB;
    uint32_t w[F::NW];
    load_lane_codes<BITS, KS>(blk, lane, w);
    const uint2 sb = *reinterpret_cast<const uint2*>(blk + F::CB + (lane >> 2) * 8);
    block_acc<BITS, KS>(w, sb, g0 + b, X, acc0, acc1);
  }
}

// ---- the same tile dot on the CUDA cores (for comparison) -------------------
//
// The group-hoisted affine dot of the Flash-MoE page ("Kernel dequant toi uu
// FMA") in fp32 on the CUDA cores, over the same record blocks: each lane
// turns its codes into floats (one byte permute and one subtraction each:
// 2^23 + q as a binary32 pattern, minus 2^23), forms sum(q * x) over its
// eight inputs per k-step for its two rows with FFMA, scales by the group's
// scale and adds bias * sum(x) once per row; the four lanes of a row quad
// are summed at the end. x is the fp32 input vector in shared memory; gs[g].y
// is the group's exact sum of inputs. No rounding of x beyond fp32.
__device__ __forceinline__ float code_f(uint32_t a, int i) {
  return __uint_as_float(__byte_perm(a, 0x4B000000u, 0x7540u | (uint32_t)i)) - 8388608.f;
}

template <int BITS, int KS>
__device__ __forceinline__ void tile_dot_fma(const unsigned char* blk0, int nblk, int g0, const float* xf,
                                             const float2* gs, float& acc0, float& acc1) {
  using F = TileFmt<BITS, KS>;
  const int lane = threadIdx.x & 31, t = lane & 3;
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 2
  for (int b = 0; b < nblk; ++b) {
    const unsigned char* blk = blk0 + (size_t)b * F::BB;
    uint32_t w[F::NW];
    load_lane_codes<BITS, KS>(blk, lane, w);
    const uint2 sb = *reinterpret_cast<const uint2*>(blk + F::CB + (lane >> 2) * 8);
    const int g = g0 + b;
    float p0 = 0.f, p1 = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a[4];
      extract_a<BITS, KS>(w, ks, a);
      const float4* xv = reinterpret_cast<const float4*>(xf + ((size_t)g * KS + ks) * 32 + 8 * t);
      const float4 x0 = xv[0], x1 = xv[1];
      const float xe[4] = {x0.x, x0.z, x1.x, x1.z};  // inputs 8t + 2i
      const float xo[4] = {x0.y, x0.w, x1.y, x1.w};  // inputs 8t + 2i + 1
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        p0 = fmaf(code_f(a[0], i), xe[i], p0);
        p0 = fmaf(code_f(a[2], i), xo[i], p0);
        p1 = fmaf(code_f(a[1], i), xe[i], p1);
        p1 = fmaf(code_f(a[3], i), xo[i], p1);
      }
    }
    const float sx = t == 0 ? gs[g].y : 0.f;
    s0 = fmaf(__uint_as_float(sb.x << 16), p0, s0);
    s0 = fmaf(__uint_as_float(sb.x & 0xFFFF0000u), sx, s0);
    s1 = fmaf(__uint_as_float(sb.y << 16), p1, s1);
    s1 = fmaf(__uint_as_float(sb.y & 0xFFFF0000u), sx, s1);
  }
  s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
  s0 += __shfl_xor_sync(0xFFFFFFFFu, s0, 2);
  s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
  s1 += __shfl_xor_sync(0xFFFFFFFFu, s1, 2);
  acc0 += s0;
  acc1 += s1;
}

// Dispatch on (bits, group) for callers with runtime values (3 bits: group
// 64 or 128 only; the host rejects 3-bit group 32).
template <typename Fn>
__device__ __forceinline__ void with_fmt(int bits, int G, Fn fn) {
  if (bits == 4) {
    if (G == 32) fn.template operator()<4, 1>();
    else if (G == 64) fn.template operator()<4, 2>();
    else fn.template operator()<4, 4>();
  } else if (bits == 3) {
    if (G == 64) fn.template operator()<3, 2>();
    else if (G == 128) fn.template operator()<3, 4>();
  } else {
    if (G == 32) fn.template operator()<2, 1>();
    else if (G == 64) fn.template operator()<2, 2>();
    else fn.template operator()<2, 4>();
  }
}

// The same dispatch with the widths fixed at compile time (a kernel built
// for routed experts at BR bits, the shared expert at BS bits, KS k-steps
// per group): only the two formats in use are compiled into it.
template <int BR, int BS, int KS, typename Fn>
__device__ __forceinline__ void with_fixed_fmt(bool routed, Fn fn) {
  if (BR == BS) {
    fn.template operator()<BR, KS>();  // one copy of the code when both widths agree
  } else {
    if (routed) fn.template operator()<BR, KS>();
    else fn.template operator()<BS, KS>();
  }
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

}  // namespace moeq
