// ffn.cuh -- moe_expert_ffn_q: gate/up dequant mat-vecs with fused SwiGLU,
// then the down dequant mat-vec, for the K routed experts and the shared
// expert of each token.
//
// Arithmetic of one row (w = q*scale + bias per group of G inputs):
//   sum_j w_j x_j = sum_g [ scale_g * sum_{j in g} q_j x_j + bias_g * sum_{j in g} x_j ]
// which is the group-summed form of fma(q, scale*x, bias*x) (Flash-MoE page,
// section "Kernel dequant toi uu FMA"): scale*x and bias*x are never formed
// per weight; scale and bias are applied once per group.
//
// Inner loop. The input vector is staged once per CTA in shared memory as
// fp16, multiplied by a power of two 2^e chosen from its max-abs value so it
// cannot overflow (exact for bf16 inputs; h loses bits below fp16's 11-bit
// significand). A 32-bit word of packed codes is split with one LOP3 per pair
// of codes into two fp16 "magic" values 1024 + q*2^s (the exponent field of
// 1024.0 above a code placed in the mantissa); the x value paired with it is
// stored pre-divided by 2^s. Mixed-precision fma.rn.f32.f16 multiplies the
// pair exactly and accumulates in fp32; the constant part 1024*x' is removed
// per half chunk with a precomputed sum. So every product q*x is exact and
// every sum is fp32.
#pragma once

#include "common.cuh"

namespace moeq {

constexpr int kFfnWarps = 8;

struct FfnParams {
  const uint8_t* experts;    // E routed records
  const uint8_t* shared;     // shared record
  size_t rec_r, rec_s;       // record bytes
  size_t off_r[6], off_s[6]; // part offsets (codes g/u/d, tables g/u/d)
  const uint16_t* x;         // [B, H] bf16
  const int32_t* idx;        // [B, K]
  float* h;                  // [B, K+1, I] (workspace)
  float* y;                  // [B, K+1, H]
  WsCtrl* ctrl;
  int H, I, E, K, G, bits_r, bits_s, B;
  int units_per_cta_gu;      // gate/up units (slot, row) per CTA
  int units_per_cta_dn;      // down units per CTA
};

// ---- shared-memory image of an input vector --------------------------------
//
// For BITS-bit codes a 32-bit word holds EPW = 32/BITS codes; it is consumed
// as EPW/2 fp16 pairs. Pair m of a word holds codes m (low half) and
// m + EPW/2 (high half), each shifted left by s = BITS*(m mod (8/BITS)) bits,
// so the image stores x[j] * 2^e / 2^s for the code it meets. A 16-byte chunk
// of codes (4 words, 128/BITS inputs) meets 4*EPW halves = EPW/2 "pieces" of
// 16 bytes; piece p of chunk c lives at 16-byte slot p*nchunk + c, so the 32
// lanes of a warp reading chunks c..c+31 of one piece touch 512 contiguous
// bytes (no bank conflicts). Per half chunk (two words) the table keeps
// C = 1024 * sum(image values) and S = 2^e * sum(x).

template <int BITS>
struct Img {
  static constexpr int EPW = 32 / BITS;     // codes per 32-bit word
  static constexpr int PAIRS = EPW / 2;     // fp16 pairs per word
  static constexpr int PIECES = EPW / 2;    // 16-byte image pieces per chunk
  static constexpr int CIN = 128 / BITS;    // inputs per chunk
  static constexpr int HC = CIN / 2;        // inputs per half chunk
  __host__ __device__ static constexpr int shift_of(int m) { return BITS * (m % (8 / BITS)); }
};

// Stage `n` inputs (fp32 through `get`) into `img` (n halves, piece-major)
// and `tab` (n / HC float2). Called by `nthreads` threads with index `tid`;
// the caller synchronises afterwards.
template <int BITS, typename Get>
__device__ void stage_image(Get get, int n, float scale, __half* img, float2* tab, int tid, int nthreads) {
  using I = Img<BITS>;
  const int nchunk = n / I::CIN, nhc = n / I::HC;
  for (int hc = tid; hc < nhc; hc += nthreads) {
    const int c = hc >> 1;
    float csum = 0.f, ssum = 0.f;
#pragma unroll
    for (int t2 = 0; t2 < 2; ++t2) {
      const int t = (hc & 1) * 2 + t2;  // word within the chunk
#pragma unroll
      for (int m = 0; m < I::PAIRS; ++m) {
        const float inv = 1.0f / (float)(1 << I::shift_of(m));
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float xv = get(c * I::CIN + t * I::EPW + m + hh * I::PAIRS);
          const __half q = __float2half_rn(xv * scale * inv);
          const int local = t * I::EPW + 2 * m + hh;  // half index within the chunk
          img[((local >> 3) * nchunk + c) * 8 + (local & 7)] = q;
          csum += 1024.f * __half2float(q);
          ssum += xv * scale;
        }
      }
    }
    tab[hc] = make_float2(csum, ssum);
  }
}

// One 32-bit word of codes against its staged pairs (packed fp16 words).
template <int BITS>
__device__ __forceinline__ float dot_word(uint32_t w, const uint32_t* xp, float acc) {
  if (BITS == 4) {
    const uint32_t w8 = w >> 8;
    acc = fma2_f16_f32((w & 0x000F000Fu) | 0x64006400u, xp[0], acc);
    acc = fma2_f16_f32((w & 0x00F000F0u) | 0x64006400u, xp[1], acc);
    acc = fma2_f16_f32((w8 & 0x000F000Fu) | 0x64006400u, xp[2], acc);
    acc = fma2_f16_f32((w8 & 0x00F000F0u) | 0x64006400u, xp[3], acc);
  } else {
    const uint32_t w8 = w >> 8;
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

// The staged inputs a 16-byte chunk of codes meets: its image pieces and the
// (C, S) sums of its two half chunks.
template <int BITS>
struct ChunkX {
  uint4 xv[Img<BITS>::PIECES];
  float4 tt;  // (C0, S0, C1, S1)
};

template <int BITS>
__device__ __forceinline__ ChunkX<BITS> load_chunk_x(int c, int nchunk, const uint4* img, const float2* tab) {
  ChunkX<BITS> X;
#pragma unroll
  for (int p = 0; p < Img<BITS>::PIECES; ++p) X.xv[p] = img[p * nchunk + c];
  X.tt = reinterpret_cast<const float4*>(tab)[c];
  return X;
}

// Contribution of one chunk of a row (16 bytes of codes `q`, (scale, bias)
// words sb0/sb1): sum over the chunk of w*x, times the image's 2^e.
template <int BITS>
__device__ __forceinline__ float chunk_dot_x(uint4 q, const ChunkX<BITS>& X, uint32_t sb0, uint32_t sb1,
                                             bool two_groups) {
  using I = Img<BITS>;
  const uint32_t* xp = reinterpret_cast<const uint32_t*>(X.xv);
  float a0 = -X.tt.x, a1 = -X.tt.z;  // remove the 1024*x' part up front
  a0 = dot_word<BITS>(q.x, xp + 0 * I::PAIRS, a0);
  a0 = dot_word<BITS>(q.y, xp + 1 * I::PAIRS, a0);
  a1 = dot_word<BITS>(q.z, xp + 2 * I::PAIRS, a1);
  a1 = dot_word<BITS>(q.w, xp + 3 * I::PAIRS, a1);
  const float s0 = bf16_bits_to_f32(sb0 & 0xFFFFu), b0 = bf16_bits_to_f32(sb0 >> 16);
  if (!two_groups) return s0 * (a0 + a1) + b0 * (X.tt.y + X.tt.w);
  const float s1 = bf16_bits_to_f32(sb1 & 0xFFFFu), b1 = bf16_bits_to_f32(sb1 >> 16);
  return s0 * a0 + b0 * X.tt.y + s1 * a1 + b1 * X.tt.w;
}

// Index of the (scale, bias) word of chunk c's first group.
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

// NR rows sharing one input image, dotted by one warp. Lane l takes chunks
// l, l+32, ...; the loads of U chunk columns of all NR rows are issued before
// any arithmetic. Returns (in lane l) row l >> (5 - log2 NR)'s dot product,
// still multiplied by the image's 2^e.
template <int BITS, int NR, int U>
__device__ __forceinline__ float rows_dot(const uint8_t* const* codes, const uint32_t* const* sbrow, int ncols, int G,
                                          const uint4* img, const float2* tab) {
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
        const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, img, tab);
#pragma unroll
        for (int r = 0; r < NR; ++r) part[r] += chunk_dot_x<BITS>(q[u][r], X, s0[u][r], s1[u][r], two);
      }
    }
  }
  return transpose_reduce<NR>(part);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

// Shared-memory plan of the gate/up kernel: images of x for the widths in use.
struct GuSmem {
  int off_img4, off_tab4, off_img2, off_tab2, bytes;
};
__host__ __device__ inline GuSmem gu_smem_plan(int H, bool need4, bool need2) {
  GuSmem s{};
  size_t o = 0;
  s.off_img4 = (int)o;
  if (need4) o += align_up((size_t)H * 2, 16);
  s.off_tab4 = (int)o;
  if (need4) o += align_up((size_t)(H / Img<4>::HC) * 8, 16);
  s.off_img2 = (int)o;
  if (need2) o += align_up((size_t)H * 2, 16);
  s.off_tab2 = (int)o;
  if (need2) o += align_up((size_t)(H / Img<2>::HC) * 8, 16);
  s.bytes = (int)o;
  return s;
}

// Persistent over units: grid (ctas, B), CTA c takes units
// [c*upc, (c+1)*upc) of token blockIdx.y, unit u = (slot u / I, row u % I);
// a warp computes the gate row and the up row of one unit together.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_gate_up(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float red[32];
  const int b = blockIdx.y;
  const bool need4 = p.bits_r == 4 || p.bits_s == 4, need2 = p.bits_r == 2 || p.bits_s == 2;
  const GuSmem sp = gu_smem_plan(p.H, need4, need2);
  pdl_wait();

  const uint16_t* xb = p.x + (size_t)b * p.H;
  float amax = 0.f;
  for (int v = threadIdx.x; v < p.H / 8; v += blockDim.x) {
    const uint4 q = reinterpret_cast<const uint4*>(xb)[v];
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int t = 0; t < 4; ++t)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[t] << 16)), fabsf(__uint_as_float(w[t] & 0xFFFF0000u))));
  }
  amax = block_max(amax, red);
  const int ex = fp16_scale_exp(amax);
  const float sc = pow2f(ex), inv_sc = pow2f(-ex);
  auto get = [&](int j) { return bf16_bits_to_f32(xb[j]); };
  if (need4) stage_image<4>(get, p.H, sc, reinterpret_cast<__half*>(smem + sp.off_img4), reinterpret_cast<float2*>(smem + sp.off_tab4), threadIdx.x, blockDim.x);
  if (need2) stage_image<2>(get, p.H, sc, reinterpret_cast<__half*>(smem + sp.off_img2), reinterpret_cast<float2*>(smem + sp.off_tab2), threadIdx.x, blockDim.x);
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
      const size_t* off = routed ? p.off_r : p.off_s;
      const int bits = routed ? p.bits_r : p.bits_s;
      const size_t rowb = (size_t)p.H * bits / 8;
      const int ng = p.H / p.G;
      const uint8_t* codes[2] = {rec + off[0] + (size_t)i * rowb, rec + off[1] + (size_t)i * rowb};
      const uint32_t* sbr[2] = {reinterpret_cast<const uint32_t*>(rec + off[3]) + (size_t)i * ng,
                                reinterpret_cast<const uint32_t*>(rec + off[4]) + (size_t)i * ng};
      float v;
      if (bits == 4)
        v = rows_dot<4, 2, 4>(codes, sbr, p.H, p.G, reinterpret_cast<const uint4*>(smem + sp.off_img4),
                              reinterpret_cast<const float2*>(smem + sp.off_tab4));
      else
        v = rows_dot<2, 2, 2>(codes, sbr, p.H, p.G, reinterpret_cast<const uint4*>(smem + sp.off_img2),
                              reinterpret_cast<const float2*>(smem + sp.off_tab2));
      const float up = __shfl_sync(0xFFFFFFFFu, v, 16);  // lanes 16..31 hold the up row
      hval = silu_f(v * inv_sc) * (up * inv_sc);
    }
    if (lane == 0) p.h[((size_t)b * (p.K + 1) + k) * p.I + i] = hval;
  }
  pdl_trigger();
}

// Shared-memory plan of the down kernel: one image of h per slot.
struct DnSmem {
  int off_img, off_tab, img_stride, tab_stride, bytes;
};
__host__ __device__ inline DnSmem dn_smem_plan(int I, int K) {
  DnSmem s{};
  s.img_stride = (int)align_up((size_t)I * 2, 16);
  s.tab_stride = (int)align_up((size_t)(I / Img<4>::HC) * 8, 16);  // 4-bit has the most half chunks
  s.off_img = 0;
  s.off_tab = s.img_stride * (K + 1);
  s.bytes = s.off_tab + s.tab_stride * (K + 1);
  return s;
}

constexpr int kDownRows = 8;  // rows of one slot per warp unit

// Persistent over units: grid (ctas, B), unit u = (slot u / (H/8), block of
// 8 rows); a warp computes 8 rows of one slot at once.
__global__ void __launch_bounds__(kFfnWarps * 32, 2) k_down(FfnParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float red[kFfnWarps][MOEQ_MAX_K + 1];
  __shared__ float s_inv[MOEQ_MAX_K + 1];
  __shared__ float s_sc[MOEQ_MAX_K + 1];
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DnSmem sp = dn_smem_plan(p.I, p.K);
  pdl_wait();

  // max |h| of every slot in one pass
  const float* hb = p.h + (size_t)b * (p.K + 1) * p.I;
  float am[MOEQ_MAX_K + 1];
#pragma unroll
  for (int k = 0; k <= MOEQ_MAX_K; ++k) am[k] = 0.f;
  for (int j = threadIdx.x; j < p.I; j += blockDim.x) {
#pragma unroll
    for (int k = 0; k <= MOEQ_MAX_K; ++k)
      if (k <= p.K) am[k] = fmaxf(am[k], fabsf(hb[(size_t)k * p.I + j]));
  }
#pragma unroll
  for (int k = 0; k <= MOEQ_MAX_K; ++k) {
    const float m = warp_max(am[k]);
    if (lane == 0 && k <= p.K) red[warp][k] = m;
  }
  __syncthreads();
  if (threadIdx.x <= p.K) {
    float m = 0.f;
    for (int w = 0; w < kFfnWarps; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    const int ex = fp16_scale_exp(m);
    s_sc[threadIdx.x] = pow2f(ex);
    s_inv[threadIdx.x] = pow2f(-ex);
  }
  __syncthreads();
  for (int k = 0; k <= p.K; ++k) {
    const float* hk = hb + (size_t)k * p.I;
    auto get = [&](int j) { return hk[j]; };
    __half* img = reinterpret_cast<__half*>(smem + sp.off_img + (size_t)k * sp.img_stride);
    float2* tab = reinterpret_cast<float2*>(smem + sp.off_tab + (size_t)k * sp.tab_stride);
    if ((k < p.K ? p.bits_r : p.bits_s) == 4)
      stage_image<4>(get, p.I, s_sc[k], img, tab, threadIdx.x, blockDim.x);
    else
      stage_image<2>(get, p.I, s_sc[k], img, tab, threadIdx.x, blockDim.x);
  }
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
      const size_t* off = routed ? p.off_r : p.off_s;
      const int bits = routed ? p.bits_r : p.bits_s;
      const size_t rowb = (size_t)p.I * bits / 8;
      const int ng = p.I / p.G;
      const uint8_t* codes[kDownRows];
      const uint32_t* sbr[kDownRows];
#pragma unroll
      for (int r = 0; r < kDownRows; ++r) {
        codes[r] = rec + off[2] + (size_t)(i0 + r) * rowb;
        sbr[r] = reinterpret_cast<const uint32_t*>(rec + off[5]) + (size_t)(i0 + r) * ng;
      }
      const uint4* img = reinterpret_cast<const uint4*>(smem + sp.off_img + (size_t)k * sp.img_stride);
      const float2* tab = reinterpret_cast<const float2*>(smem + sp.off_tab + (size_t)k * sp.tab_stride);
      const float v = bits == 4 ? rows_dot<4, kDownRows, 1>(codes, sbr, p.I, p.G, img, tab)
                                : rows_dot<2, kDownRows, 1>(codes, sbr, p.I, p.G, img, tab);
      yval = v * s_inv[k];
    }
    if ((lane & 3) == 0) p.y[((size_t)b * (p.K + 1) + k) * p.H + i0 + (lane >> 2)] = yval;
  }
  pdl_trigger();
}

}  // namespace moeq
