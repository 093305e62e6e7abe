// dqdot.cuh -- the group-affine dequant dot product shared by every kernel.
//
// One row of a code matrix against an input vector x (w = q*scale + bias per
// group of G consecutive inputs):
//   sum_j w_j x_j = sum_g [ scale_g * sum_{j in g} q_j x_j + bias_g * sum_{j in g} x_j ]
// i.e. the group-summed form of the Flash-MoE page's fma(q, scale*x, bias*x)
// (section "Kernel dequant toi uu FMA"): scale and bias are applied once per
// group, never per weight.
//
// The input vector is staged once in shared memory as an fp16 "image". A
// 16-byte chunk of codes (4 words, CIN = 128/BITS inputs) meets CIN image
// values; every chunk has its own power-of-two scale 2^e, picked from the
// chunk's max |x| so that no image value exceeds 2^15 (exact for bf16 inputs;
// fp32 inputs keep fp16's 11 significant bits).
//
// A 32-bit word of codes holds EPW = 32/BITS codes and is consumed as EPW/2
// fp16 pairs: one LOP3 turns codes m and m + EPW/2 into the halves of
// (w & mask_m) | 0x64006400, i.e. 1024 + q*2^s with s = BITS*(m mod (8/BITS))
// (the exponent field of 1024.0 sits above the code in the mantissa). The
// image holds x * 2^e / 2^s for that code, so a mixed-precision
// fma.rn.f32.f16 forms (1024 + q*2^s) * x * 2^e / 2^s exactly in fp32 and
// accumulates in fp32. Per half chunk the table keeps C = 1024 * sum(image)
// (subtracted up front) and S = sum(x) (for the bias term).
//
// Layout, for a vector of n inputs (nchunk = n / CIN chunks):
//   img  uint4  [PIECES][nchunk]   piece p of chunk c at p*nchunk + c, so the
//                                  lanes of a warp reading consecutive chunks
//                                  of one piece touch contiguous bytes
//   tab  float4 [nchunk]           (C0, C1, S0, S1) of the two half chunks
//   inv  float  [nchunk]           2^-e of the chunk
#pragma once

#include "common.cuh"

namespace moeq {

template <int BITS>
struct Img {
  static constexpr int EPW = 32 / BITS;   // codes per 32-bit word
  static constexpr int PAIRS = EPW / 2;   // fp16 pairs per word
  static constexpr int PIECES = EPW / 2;  // 16-byte image pieces per chunk
  static constexpr int CIN = 128 / BITS;  // inputs per chunk
  __host__ __device__ static constexpr int shift_of(int m) { return BITS * (m % (8 / BITS)); }
};

// Shared-memory footprint of one staged vector.
__host__ __device__ inline size_t img_bytes(int n) { return (size_t)n * 2; }
__host__ __device__ inline size_t tab_bytes(int n, int bits) { return (size_t)(n * bits / 128) * 16; }
__host__ __device__ inline size_t inv_bytes(int n, int bits) { return (size_t)(n * bits / 128) * 4; }

struct ImgRef {
  uint4* img;
  float4* tab;
  float* inv;
};

// Stage chunk c from its CIN input values v (fp32, final values).
template <int BITS>
__device__ __forceinline__ void stage_chunk(const float* v, int c, int nchunk, ImgRef R) {
  using I = Img<BITS>;
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < I::CIN; ++j) amax = fmaxf(amax, fabsf(v[j]));
  const int e = fp16_scale_exp(amax);
  const float sc = pow2f(e);
  float C[2] = {0.f, 0.f}, S[2] = {0.f, 0.f};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint32_t packed[I::PAIRS];
#pragma unroll
    for (int m = 0; m < I::PAIRS; ++m) {
      const float lo = v[t * I::EPW + m], hi = v[t * I::EPW + m + I::PAIRS];
      const float s = sc * (1.0f / (float)(1 << I::shift_of(m)));
      const __half hl = __float2half_rn(lo * s), hh = __float2half_rn(hi * s);
      packed[m] = (uint32_t)__half_as_ushort(hl) | ((uint32_t)__half_as_ushort(hh) << 16);
      C[t >> 1] += 1024.f * (__half2float(hl) + __half2float(hh));
      S[t >> 1] += lo + hi;
    }
#pragma unroll
    for (int q = 0; q < I::PAIRS / 4; ++q)
      R.img[(t * (I::PAIRS / 4) + q) * nchunk + c] =
          make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
  }
  R.tab[c] = make_float4(C[0], C[1], S[0], S[1]);
  R.inv[c] = pow2f(-e);
}

// CIN bf16 inputs (global or shared memory, 16-byte aligned) -> fp32 values.
template <int BITS>
__device__ __forceinline__ void load_bf16_chunk(const uint16_t* src, float* v) {
#pragma unroll
  for (int q = 0; q < Img<BITS>::CIN / 8; ++q) {
    const uint4 w = reinterpret_cast<const uint4*>(src)[q];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(ww[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
  }
}

// CIN fp32 inputs written by other CTAs of this grid or an earlier kernel
// (read at L2, 16-byte aligned).
template <int BITS>
__device__ __forceinline__ void load_f32_chunk_cg(const float* src, float* v) {
#pragma unroll
  for (int q = 0; q < Img<BITS>::CIN / 4; ++q) {
    const float4 f = __ldcg(reinterpret_cast<const float4*>(src) + q);
    v[4 * q] = f.x;
    v[4 * q + 1] = f.y;
    v[4 * q + 2] = f.z;
    v[4 * q + 3] = f.w;
  }
}

// One 32-bit word of codes against its staged pairs (packed fp16 words).
template <int BITS>
__device__ __forceinline__ float dot_word(uint32_t w, const uint32_t* xp, float acc) {
  const uint32_t w8 = w >> 8;
  if (BITS == 4) {
    acc = fma2_f16_f32((w & 0x000F000Fu) | 0x64006400u, xp[0], acc);
    acc = fma2_f16_f32((w & 0x00F000F0u) | 0x64006400u, xp[1], acc);
    acc = fma2_f16_f32((w8 & 0x000F000Fu) | 0x64006400u, xp[2], acc);
    acc = fma2_f16_f32((w8 & 0x00F000F0u) | 0x64006400u, xp[3], acc);
  } else {
    acc = fma2_f16_f32((w & 0x00030003u) | 0x64006400u, xp[0], acc);
    acc = fma2_f16_f32((w & 0x000C000Cu) | 0x64006400u, xp[1], acc);
    acc = fma2_f16_f32((w & 0x00300030u) | 0x64006400u, xp[2], acc);
    acc = fma2_f16_f32((w & 0x00C000C0u) | 0x64006400u, xp[3], acc);
    acc = fma2_f16_f32((w8 & 0x00030003u) | 0x64006400u, xp[4], acc);
    acc = fma2_f16_f32((w8 & 0x000C000Cu) | 0x64006400u, xp[5], acc);
    acc = fma2_f16_f32((w8 & 0x00300030u) | 0x64006400u, xp[6], acc);
    acc = fma2_f16_f32((w8 & 0x00C000C0u) | 0x64006400u, xp[7], acc);
  }
  return acc;
}

// What one chunk of codes meets: its image pieces, table entry and 2^-e.
template <int BITS>
struct ChunkX {
  uint4 xv[Img<BITS>::PIECES];
  float4 tt;  // (C0, C1, S0, S1)
  float inv;
};

template <int BITS>
__device__ __forceinline__ ChunkX<BITS> load_chunk_x(int c, int nchunk, const ImgRef& R) {
  ChunkX<BITS> X;
#pragma unroll
  for (int p = 0; p < Img<BITS>::PIECES; ++p) X.xv[p] = R.img[p * nchunk + c];
  X.tt = R.tab[c];
  X.inv = R.inv[c];
  return X;
}

// Contribution of one chunk of a row: 16 bytes of codes q and the (scale,
// bias) words of its group(s). Returns sum over the chunk of w*x.
template <int BITS>
__device__ __forceinline__ float chunk_dot_x(uint4 q, const ChunkX<BITS>& X, uint32_t sb0, uint32_t sb1,
                                             bool two_groups) {
  using I = Img<BITS>;
  const uint32_t* xp = reinterpret_cast<const uint32_t*>(X.xv);
  float a0 = -X.tt.x, a1 = -X.tt.y;  // remove the 1024*image part up front
  a0 = dot_word<BITS>(q.x, xp + 0 * I::PAIRS, a0);
  a0 = dot_word<BITS>(q.y, xp + 1 * I::PAIRS, a0);
  a1 = dot_word<BITS>(q.z, xp + 2 * I::PAIRS, a1);
  a1 = dot_word<BITS>(q.w, xp + 3 * I::PAIRS, a1);
  const float s0 = bf16_bits_to_f32(sb0 & 0xFFFFu), b0 = bf16_bits_to_f32(sb0 >> 16);
  if (!two_groups) return s0 * ((a0 + a1) * X.inv) + b0 * (X.tt.z + X.tt.w);
  const float s1 = bf16_bits_to_f32(sb1 & 0xFFFFu), b1 = bf16_bits_to_f32(sb1 >> 16);
  return (s0 * a0 + s1 * a1) * X.inv + b0 * X.tt.z + b1 * X.tt.w;
}

// Index of the (scale, bias) word of chunk c's first group; a chunk spans two
// groups only for 2-bit codes with group 32.
template <int BITS>
__device__ __forceinline__ int chunk_group(int c, int G, bool two) {
  return two ? 2 * c : (c * Img<BITS>::CIN) / G;
}

// Sum over 32 lanes of NR per-lane partials (one per row), transposed so
// that no value is reduced twice: after log2(NR) exchange stages each lane
// holds one row's partial summed over its partner lanes, then a plain
// butterfly finishes. Lane l ends with the total of row l >> (5 - log2 NR).
template <int NR>
__device__ __forceinline__ float transpose_reduce(float (&v)[NR]) {
  const int lane = threadIdx.x & 31;
  constexpr int LOG = NR == 1 ? 0 : NR == 2 ? 1 : NR == 4 ? 2 : NR == 8 ? 3 : 4;
  static_assert((1 << LOG) == NR && NR <= 16, "NR must be a power of two <= 16");
#pragma unroll
  for (int s = 0; s < LOG; ++s) {
    const int o = 16 >> s;
    const int half = NR >> (s + 1);
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float keep = upper ? v[j + half] : v[j];
      const float send = upper ? v[j] : v[j + half];
      v[j] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  float t = v[0];
#pragma unroll
  for (int o = 16 >> LOG; o > 0; o >>= 1) t += __shfl_xor_sync(0xFFFFFFFFu, t, o);
  return t;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

}  // namespace moeq
