// pack.cuh -- moe_pack_q / moe_pack_expert: one u8 code per byte -> b-bit
// fields, low bits first, plus (scale, bias) bf16 pairs per (row, group).
#pragma once

#include "common.cuh"

namespace moeq {

// Where row r of a packed matrix goes: rows come in blocks of `rpb` rows;
// block r / rpb starts at base + (r / rpb) * blk_stride and its rows are
// row_stride apart. A plain row-major matrix is one block.
struct RowPlace {
  unsigned char* base;
  int rpb;
  size_t row_stride, blk_stride;
  __device__ __forceinline__ unsigned char* row(int r) const {
    return base + (size_t)(r / rpb) * blk_stride + (size_t)(r % rpb) * row_stride;
  }
};

// 4 codes in the bytes of v -> 4 nibbles (16 bits), element order kept.
__device__ __forceinline__ uint32_t nib4(uint32_t v) {
  return (v & 0xFu) | ((v >> 4) & 0xF0u) | ((v >> 8) & 0xF00u) | ((v >> 12) & 0xF000u);
}
// 4 codes in the bytes of v -> 4 two-bit fields (8 bits).
__device__ __forceinline__ uint32_t crumb4(uint32_t v) {
  return (v & 0x3u) | ((v >> 6) & 0xCu) | ((v >> 12) & 0x30u) | ((v >> 18) & 0xC0u);
}

// One thread writes one 16-byte output chunk: 32 codes at 4 bits, 64 at 2
// bits. Rows are whole chunks (cols*BITS/8 is a multiple of 16).
template <int BITS>
__global__ void __launch_bounds__(256) k_pack_codes(const uint8_t* __restrict__ codes, int64_t nchunks, int cpr,
                                                    RowPlace dst, WsCtrl* ctrl) {
  constexpr int CODES = 128 / BITS;  // codes per output chunk
  uint32_t bad = 0;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < nchunks; c += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + c * CODES);
    uint32_t out[4];
    if (BITS == 4) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint4 v = src[h];
        bad |= (v.x | v.y | v.z | v.w) & 0xF0F0F0F0u;
        out[2 * h + 0] = nib4(v.x) | (nib4(v.y) << 16);
        out[2 * h + 1] = nib4(v.z) | (nib4(v.w) << 16);
      }
    } else {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint4 v = src[h];
        bad |= (v.x | v.y | v.z | v.w) & 0xFCFCFCFCu;
        out[h] = crumb4(v.x) | (crumb4(v.y) << 8) | (crumb4(v.z) << 16) | (crumb4(v.w) << 24);
      }
    }
    const int r = (int)(c / cpr), cc = (int)(c % cpr);
    reinterpret_cast<uint4*>(dst.row(r))[cc] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (bad) set_error(ctrl, MOE_ERR_RANGE);
}

// 3 bits: one thread writes 48 output bytes, 128 codes as one little-endian
// bit string (code j at bits 3j..3j+2; a code may straddle two bytes or two
// words). Rows are whole 128-code runs (cols % 128 == 0).
__global__ void __launch_bounds__(256) k_pack_codes3(const uint8_t* __restrict__ codes, int64_t nruns, int rpr,
                                                     RowPlace dst, WsCtrl* ctrl) {
  uint32_t bad = 0;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < nruns; c += (int64_t)gridDim.x * blockDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + c * 128);
    uint32_t out[12];
#pragma unroll
    for (int i = 0; i < 12; ++i) out[i] = 0u;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const uint4 v = src[h];
      const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const uint32_t code = (vv[q >> 2] >> (8 * (q & 3))) & 0xFFu;
        bad |= code & 0xF8u;
        const int bit = 3 * (16 * h + q);
        out[bit >> 5] |= (code & 7u) << (bit & 31);
        if ((bit & 31) > 29) out[(bit >> 5) + 1] |= (code & 7u) >> (32 - (bit & 31));
      }
    }
    const int r = (int)(c / rpr), cc = (int)(c % rpr);
    uint4* o = reinterpret_cast<uint4*>(dst.row(r) + (size_t)cc * 48);
    o[0] = make_uint4(out[0], out[1], out[2], out[3]);
    o[1] = make_uint4(out[4], out[5], out[6], out[7]);
    o[2] = make_uint4(out[8], out[9], out[10], out[11]);
  }
  if (bad) set_error(ctrl, MOE_ERR_RANGE);
}

// (scale, bias) -> one 32-bit pair, scale in the low half (first in memory);
// ngr pairs per row.
__global__ void __launch_bounds__(256) k_pack_sb(const uint16_t* __restrict__ scale, const uint16_t* __restrict__ bias,
                                                 int64_t n, int ngr, RowPlace dst) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / ngr), g = (int)(i % ngr);
    reinterpret_cast<uint32_t*>(dst.row(r))[g] = (uint32_t)scale[i] | ((uint32_t)bias[i] << 16);
  }
}

// ---- expert records: tiles of 16 rows in mma fragment order ---------------

// Where local row rho of tile T comes from: gate/up tiles (split 8) take rows
// 8T..8T+7 of matrix 0 then rows 8T..8T+7 of matrix 1; down tiles (split 16)
// take rows 16T..16T+15 of matrix 0. Every matrix has C inputs per row.
struct TileSrc {
  const uint8_t* codes[2];
  const uint16_t* scale[2];
  const uint16_t* bias[2];
  int split;
  __device__ __forceinline__ int mat(int rho) const { return (split == 8 && rho >= 8) ? 1 : 0; }
  __device__ __forceinline__ int row(int T, int rho) const { return split == 8 ? 8 * T + (rho & 7) : 16 * T + rho; }
};

// One thread per (tile, group, lane, k-step): the lane's codes of local rows
// gid and gid+8 for inputs 32m+8t .. 32m+8t+7 of the group's k-step m.
// 4 bits: two words, input 8t+i of a row at nibble i. 2 bits: one word, input
// 8t+2i of row gid at bits 8i, of row gid+8 at 8i+2, input 8t+2i+1 of row gid
// at 8i+4, of row gid+8 at 8i+6.
template <int BITS>
__global__ void __launch_bounds__(256) k_pack_tile_codes(TileSrc src, int ntiles, int C, int G, unsigned char* dst,
                                                         uint32_t tile_bytes, uint32_t blk_bytes, WsCtrl* ctrl) {
  constexpr int W = BITS == 4 ? 8 : 4;
  const int KS = G / 32, ng = C / G;
  const int64_t total = (int64_t)ntiles * ng * 32 * KS;
  uint32_t bad = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(i % KS);
    const int L = (int)((i / KS) % 32);
    const int g = (int)((i / (KS * 32)) % ng);
    const int T = (int)(i / ((int64_t)KS * 32 * ng));
    const int gid = L >> 2, t = L & 3;
    const int col = g * G + 32 * j + 8 * t;
    uint32_t c[2][2];  // [local row gid / gid+8][two words of 4 codes]
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rho = gid + 8 * h;
      const uint2 v = *reinterpret_cast<const uint2*>(src.codes[src.mat(rho)] + (size_t)src.row(T, rho) * C + col);
      c[h][0] = v.x;
      c[h][1] = v.y;
      bad |= (v.x | v.y) & (BITS == 4 ? 0xF0F0F0F0u : 0xFCFCFCFCu);
    }
    unsigned char* out = dst + (size_t)T * tile_bytes + (size_t)g * blk_bytes + (size_t)L * (KS * W) + (size_t)j * W;
    if (BITS == 4) {
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t x = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) x |= ((c[h][q >> 2] >> (8 * (q & 3))) & 0xFu) << (4 * q);
        w[h] = x;
      }
      *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
    } else {
      uint32_t x = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int i = q >> 1, odd = q & 1;  // input 2i + odd of the eight
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t code = (c[h][q >> 2] >> (8 * (q & 3))) & 0x3u;
          x |= code << (8 * i + 4 * odd + 2 * h);
        }
      }
      *reinterpret_cast<uint32_t*>(out) = x;
    }
  }
  if (bad) set_error(ctrl, MOE_ERR_RANGE);
}

// 3 bits: one thread per (tile, group, lane, pair of k-steps 2p, 2p+1). The
// low two bits of each code go to the lane's 2-bit plane word of each k-step
// (the 2-bit layout above); the third bits of both k-steps share one word of
// the third-bit plane: bit 8i + 4*(k-step & 1) + r is the third bit of byte
// i of A register r (r = 2*odd + h: input 8t+2i+odd of local row gid + 8h).
__global__ void __launch_bounds__(256) k_pack_tile_codes3(TileSrc src, int ntiles, int C, int G, unsigned char* dst,
                                                          uint32_t tile_bytes, uint32_t blk_bytes, WsCtrl* ctrl) {
  const int KS = G / 32, ng = C / G, NP = KS / 2;
  const int64_t total = (int64_t)ntiles * ng * 32 * NP;
  uint32_t bad = 0;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int pp = (int)(i % NP);
    const int L = (int)((i / NP) % 32);
    const int g = (int)((i / (NP * 32)) % ng);
    const int T = (int)(i / ((int64_t)NP * 32 * ng));
    const int gid = L >> 2, t = L & 3;
    unsigned char* blk = dst + (size_t)T * tile_bytes + (size_t)g * blk_bytes;
    uint32_t hi = 0;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 2 * pp + e;
      const int col = g * G + 32 * j + 8 * t;
      uint32_t c[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rho = gid + 8 * h;
        const uint2 v = *reinterpret_cast<const uint2*>(src.codes[src.mat(rho)] + (size_t)src.row(T, rho) * C + col);
        c[h][0] = v.x;
        c[h][1] = v.y;
        bad |= (v.x | v.y) & 0xF8F8F8F8u;
      }
      uint32_t lo = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int ii = q >> 1, odd = q & 1;  // input 2ii + odd of the eight
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t code = (c[h][q >> 2] >> (8 * (q & 3))) & 0x7u;
          const int r = 2 * odd + h;
          lo |= (code & 3u) << (8 * ii + 2 * r);
          hi |= (code >> 2) << (8 * ii + 4 * e + r);
        }
      }
      *reinterpret_cast<uint32_t*>(blk + (size_t)L * (KS * 4) + (size_t)j * 4) = lo;
    }
    *reinterpret_cast<uint32_t*>(blk + (size_t)32 * KS * 4 + (size_t)L * (KS * 2) + (size_t)pp * 4) = hi;
  }
  if (bad) set_error(ctrl, MOE_ERR_RANGE);
}

// One thread per (tile, group, gid): the (scale, bias) pairs of local rows
// gid and gid+8 after the block's codes.
__global__ void __launch_bounds__(256) k_pack_tile_sb(TileSrc src, int ntiles, int C, int G, unsigned char* dst,
                                                      uint32_t tile_bytes, uint32_t blk_bytes, uint32_t code_bytes) {
  const int ng = C / G;
  const int64_t total = (int64_t)ntiles * ng * 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int gid = (int)(i % 8);
    const int g = (int)((i / 8) % ng);
    const int T = (int)(i / (8 * ng));
    uint32_t pr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rho = gid + 8 * h, m = src.mat(rho);
      const size_t at = (size_t)src.row(T, rho) * ng + g;
      pr[h] = (uint32_t)src.scale[m][at] | ((uint32_t)src.bias[m][at] << 16);
    }
    *reinterpret_cast<uint2*>(dst + (size_t)T * tile_bytes + (size_t)g * blk_bytes + code_bytes + (size_t)gid * 8) =
        make_uint2(pr[0], pr[1]);
  }
}

// ---- quantisation: weights -> codes, scale, bias ---------------------------

// Min-max group-affine quantisation, one warp per (row, group): lo and hi
// are the group's extreme weights; scale = bf16((hi - lo) / (2^BITS - 1)),
// bias = bf16(lo); q = clamp(rint((w - bias) / scale), 0, 2^BITS - 1), 0 when
// the bf16 scale is 0 (the affine form w ~ q*scale + bias of the Flash-MoE
// page, "Kernel dequant toi uu FMA"). Every step is one binary32 operation
// rounded to nearest even (no contraction), so the codes are reproducible.
// A non-finite weight sets MOE_ERR_RANGE and its group is written as zeros.
template <int GPL>  // weights per lane: group / 32
__global__ void __launch_bounds__(256) k_quantize(const void* __restrict__ w, int in_bf16, int64_t ngroups, int ng,
                                                  int cols, int bits, uint8_t* __restrict__ codes,
                                                  uint16_t* __restrict__ scale, uint16_t* __restrict__ bias,
                                                  WsCtrl* ctrl) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float levels = (float)((1 << bits) - 1);
  for (int64_t gi = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); gi < ngroups; gi += nwarps) {
    const int64_t r = gi / ng;
    const int g = (int)(gi % ng);
    const int64_t at = r * cols + (int64_t)g * (32 * GPL) + lane * GPL;
    float v[GPL];
#pragma unroll
    for (int i = 0; i < GPL; ++i)
      v[i] = in_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(w)[at + i])
                     : reinterpret_cast<const float*>(w)[at + i];
    bool fin = true;
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int i = 0; i < GPL; ++i) {
      fin = fin && isfinite(v[i]);
      lo = fminf(lo, v[i]);
      hi = fmaxf(hi, v[i]);
    }
    fin = __all_sync(0xFFFFFFFFu, fin);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    uint16_t sbits = 0, bbits = 0;
    uint8_t q[GPL];
#pragma unroll
    for (int i = 0; i < GPL; ++i) q[i] = 0;
    if (fin) {
      const float s32 = __fdiv_rn(__fsub_rn(hi, lo), levels);
      sbits = f32_to_bf16_bits(s32);
      bbits = f32_to_bf16_bits(lo);
      const float sf = bf16_bits_to_f32(sbits), bf = bf16_bits_to_f32(bbits);
      if (sf != 0.f) {
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
          const float t = rintf(__fdiv_rn(__fsub_rn(v[i], bf), sf));
          q[i] = (uint8_t)(t < 0.f ? 0.f : (t > levels ? levels : t));
        }
      }
    } else if (lane == 0) {
      set_error(ctrl, MOE_ERR_RANGE);
    }
#pragma unroll
    for (int i = 0; i < GPL; ++i) codes[at + i] = q[i];
    if (lane == 0) {
      scale[gi] = sbits;
      bias[gi] = bbits;
    }
  }
}

}  // namespace moeq
