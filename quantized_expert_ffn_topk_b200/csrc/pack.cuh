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

}  // namespace moeq
