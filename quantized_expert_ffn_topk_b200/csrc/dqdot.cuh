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

// Staging is done 16 inputs per thread: a chunk is split into TPC = CIN/16
// segments held by TPC adjacent lanes (4-bit: 2 lanes of two words each;
// 2-bit: 4 lanes of one word each). The lanes agree on the chunk's scale and
// table entry through shuffles. Every lane of the warp must call the staging
// functions together; lanes without a segment pass active = false.
template <int BITS>
struct Seg {
  static constexpr int TPC = Img<BITS>::CIN / 16;  // lanes per chunk
  static constexpr int WORDS = 16 / Img<BITS>::EPW;  // words per segment (2 or 1)
};

// Stage segment s of chunk c from its 16 input values v (fp32, final values).
template <int BITS>
__device__ __forceinline__ void stage_seg(const float (&v)[16], int c, int s, int nchunk, ImgRef R, bool active) {
  using I = Img<BITS>;
  using SG = Seg<BITS>;
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
#pragma unroll
  for (int o = 1; o < SG::TPC; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const int e = fp16_scale_exp(amax);
  const float sc = pow2f(e);
  float C = 0.f, S = 0.f;
#pragma unroll
  for (int tw = 0; tw < SG::WORDS; ++tw) {
    const int t = s * SG::WORDS + tw;  // word within the chunk
    uint32_t packed[I::PAIRS];
#pragma unroll
    for (int m = 0; m < I::PAIRS; ++m) {
      const float lo = v[tw * I::EPW + m], hi = v[tw * I::EPW + m + I::PAIRS];
      const float f = sc * (1.0f / (float)(1 << I::shift_of(m)));
      const __half hl = __float2half_rn(lo * f), hh = __float2half_rn(hi * f);
      packed[m] = (uint32_t)__half_as_ushort(hl) | ((uint32_t)__half_as_ushort(hh) << 16);
      C += 1024.f * (__half2float(hl) + __half2float(hh));
      S += lo + hi;
    }
    if (active) {
#pragma unroll
      for (int q = 0; q < I::PAIRS / 4; ++q)
        R.img[(t * (I::PAIRS / 4) + q) * nchunk + c] =
            make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
    }
  }
  // half-chunk sums: 4-bit segments are half chunks; 2-bit half chunks are two segments
  if (BITS == 2) {
    C += __shfl_xor_sync(0xFFFFFFFFu, C, 1);
    S += __shfl_xor_sync(0xFFFFFFFFu, S, 1);
  }
  const int other = BITS == 4 ? 1 : 2;  // lane offset of the chunk's second half
  const float C1 = __shfl_xor_sync(0xFFFFFFFFu, C, other), S1 = __shfl_xor_sync(0xFFFFFFFFu, S, other);
  if (active && s == 0) {
    R.tab[c] = make_float4(C, C1, S, S1);
    R.inv[c] = pow2f(-e);
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

// 16 fp32 inputs written by other CTAs or an earlier kernel (read at L2).
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

// One warp stages segments [32*gi, 32*gi + 32) of a vector of n inputs
// (n a multiple of CIN); get(j0, v) fills the 16 values starting at input j0.
template <int BITS, typename Get>
__device__ __forceinline__ void stage_group(Get get, int n, ImgRef R, int gi, int lane) {
  constexpr int TPC = Seg<BITS>::TPC;
  const int t = gi * 32 + lane;
  const bool active = t < n / 16;
  float v[16];
  if (active) {
    get(t * 16, v);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = 0.f;
  }
  stage_seg<BITS>(v, t / TPC, t % TPC, n / Img<BITS>::CIN, R, active);
}

// Stage a whole vector with nthr threads (a multiple of 32).
template <int BITS, typename Get>
__device__ __forceinline__ void stage_vector(Get get, int n, ImgRef R, int tid, int nthr) {
  for (int gi = tid >> 5; gi * 32 < n / 16; gi += nthr >> 5) stage_group<BITS>(get, n, R, gi, tid & 31);
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
