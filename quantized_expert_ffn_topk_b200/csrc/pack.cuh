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

}  // namespace moeq
