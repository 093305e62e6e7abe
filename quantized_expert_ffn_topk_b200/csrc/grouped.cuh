// grouped.cuh -- moe_expert_ffn_q for a batch of tokens, grouped by expert:
// each active expert's weights are read once per step for all the tokens
// routed to it (the batched-decode token grouping; the pages themselves run
// one token at a time).
//
//   k_group           stable counting sort of the (token, slot) picks by
//                     expert id: cnt, off, list, and the active experts
//   k_stage_batch     the input image of every token (x, or h per slot) in
//                     the workspace, so that a tile can be applied to
//                     several tokens without restaging
//   k_gate_up_grp     unit = (expert, gate/up tile): the tile is read once;
//                     four tokens share each mma (columns 2t, 2t+1 carry
//                     token t's hi and lo planes); h per (token, slot)
//   k_down_grp        unit = (expert, down tile): y per (token, slot)
//
// The work items of a step are [the shared expert's token chunks, the
// active routed experts' chunks in increasing id]; the shared expert serves
// every token (slot K).
#pragma once

#include "common.cuh"
#include "ffn.cuh"
#include "tiledot.cuh"

namespace moeq {

constexpr int kGrpWarps = 8;
// (measured at 32 and 128 tokens per step on the 4-bit layer: 3 CTAs per SM
// with 4 blocks in flight per warp beat 4 x 2, 4 x 3, 3 x 3, 3 x 5, 2 x 6 and
// 2 x 8)
#ifndef MOEQ_GRP_CTAS
#define MOEQ_GRP_CTAS 3
#endif
#ifndef MOEQ_GRP_INFLIGHT
#define MOEQ_GRP_INFLIGHT 4
#endif
constexpr int kGrpCtasPerSm = MOEQ_GRP_CTAS;        // resident CTAs per SM (85 registers a thread at 3)
constexpr int kGrpInFlight = MOEQ_GRP_INFLIGHT;     // blocks whose loads a warp keeps in flight
// Pieces of a tile (warps that share a unit, a part of its groups each): a
// down tile has a quarter of a gate/up tile's groups, so its units are
// dealt whole to one warp and a round carries more of them.
#ifndef MOEQ_GRP_PIECES_GU
#define MOEQ_GRP_PIECES_GU 4
#endif
#ifndef MOEQ_GRP_PIECES_DN
#define MOEQ_GRP_PIECES_DN 1
#endif
constexpr int kGrpPiecesGu = MOEQ_GRP_PIECES_GU;
constexpr int kGrpPiecesDn = MOEQ_GRP_PIECES_DN;
static_assert(kGrpWarps % kGrpPiecesGu == 0 && kGrpWarps % kGrpPiecesDn == 0, "whole units per round");
constexpr int kGrpMaxTok = 64;                      // tokens of one work item at most
// (work items of 16 or 8 of the shared expert's tokens measured no faster
// than 64 at 32 and 128 tokens per step once units are dealt on demand)
#ifndef MOEQ_GRP_SHARED_TOK
#define MOEQ_GRP_SHARED_TOK 64
#endif
constexpr int kGrpSharedTok = MOEQ_GRP_SHARED_TOK;  // tokens of one of the shared expert's work items
static_assert(kGrpSharedTok <= kGrpMaxTok, "work items hold kGrpMaxTok tokens at most");
constexpr int kGrpSharedItems = (MOEQ_MAX_B + kGrpSharedTok - 1) / kGrpSharedTok;  // the shared expert's work items at most

// A routed expert with more than kGrpMaxTok entries (popular experts of a
// large batch, or forced picks that repeat an expert within a token) is split
// into several chunks; a chunk is one work item. The shared expert serves
// every token: ceil(B / kGrpMaxTok) work items of consecutive tokens.
constexpr int kGrpExtraChunks = (MOEQ_MAX_B * MOEQ_MAX_K) / kGrpMaxTok;
struct GrpWs {
  int* cnt;   // [E]
  int* off;   // [E + 1]
  int* list;  // [B*K]: entries b*K + k grouped by expert, in entry order
  int* act;   // [E + kGrpExtraChunks][3]: (expert, its first entry in list, entries) per chunk, by expert id
  int* nact;  // [3]: chunks, then the next unit of the gate/up and of the down kernel (0 after grouping)
};

struct GrpParams {
  FfnParams f;
  GrpWs g;
  unsigned char* img;   // per-source images: x [B] (gate/up) or h [B][K+1] (down)
  int img_stride;       // bytes between consecutive images
  int img_gs_off;       // byte offset of the gs array within an image
  int tps;              // tiles per expert (I/8 gate/up, H/16 down)
  int max_units;        // (shared work items + most routed work items) * tps
  int nsh;              // the shared expert's work items: ceil(B / kGrpMaxTok)
};

// ---- grouping -------------------------------------------------------------

// One CTA. Picks outside [0, E) set MOE_ERR_INDEX, are left out of every
// group, and get a zero output slot here.
__global__ void __launch_bounds__(256) k_group(const int32_t* idx, int B, int K, int E, int H, GrpWs g, float* y,
                                               WsCtrl* ctrl) {
  extern __shared__ int s_cnt[];  // [max(E + 1, B*K)]: counts, then the picks
  pdl_wait();
  const int n = B * K;
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) {
      atomicAdd(&s_cnt[e], 1);
    } else {
      set_error(ctrl, MOE_ERR_INDEX);
      float* yk = y + ((size_t)(i / K) * (K + 1) + (i % K)) * H;
      for (int h = 0; h < H; ++h) yk[h] = 0.f;
    }
  }
  __syncthreads();
  // offsets of each expert's entries and of its chunks: exclusive scans over
  // the experts, each thread taking a contiguous range of them
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
  int sc = 0, sk = 0;
  for (int e = e0; e < e1; ++e) {
    sc += s_cnt[e];
    sk += (s_cnt[e] + kGrpMaxTok - 1) / kGrpMaxTok;
  }
  __shared__ int s_wc[32], s_wk[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int ic = sc, ik = sk;  // inclusive scans within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int tc = __shfl_up_sync(0xFFFFFFFFu, ic, o), tk = __shfl_up_sync(0xFFFFFFFFu, ik, o);
    if (lane >= o) {
      ic += tc;
      ik += tk;
    }
  }
  if (lane == 31) {
    s_wc[warp] = ic;
    s_wk[warp] = ik;
  }
  __syncthreads();
  int oc = ic - sc, ok = ik - sk;
  for (int w = 0; w < warp; ++w) {
    oc += s_wc[w];
    ok += s_wk[w];
  }
  for (int e = e0; e < e1; ++e) {
    const int c = s_cnt[e];
    g.cnt[e] = c;
    g.off[e] = oc;
    for (int c0 = 0; c0 < c; c0 += kGrpMaxTok, ++ok) {
      g.act[3 * ok] = e;
      g.act[3 * ok + 1] = oc + c0;
      g.act[3 * ok + 2] = min(kGrpMaxTok, c - c0);
    }
    oc += c;
  }
  if (threadIdx.x == 0) {
    int tc = 0, tk = 0;
    for (int w = 0; w < nw; ++w) {
      tc += s_wc[w];
      tk += s_wk[w];
    }
    g.off[E] = tc;
    g.nact[0] = tk;
    g.nact[1] = 0;
    g.nact[2] = 0;
  }
  __syncthreads();
  // each entry's rank among the earlier entries of its expert (a stable
  // order), from a copy of the picks in the shared memory the counts used
  // (sized for max(E + 1, B*K) ints by the host)
  int* s_idx = s_cnt;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s_idx[i] = idx[i];
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = s_idx[i];
    if (e < 0 || e >= E) continue;
    int r = 0;
    for (int j = 0; j < i; ++j) r += s_idx[j] == e;
    g.list[g.off[e] + r] = i;
  }
  pdl_trigger();
}

// Images of B tokens' x (grid B) or of every (token, slot)'s h (grid
// (B, K+1)): image b (or b*(K+1)+k) at img + index * stride.
__global__ void __launch_bounds__(256) k_stage_batch(const void* src, int is_h, int n, int G, unsigned char* img,
                                                     int stride, int gs_off) {
  pdl_wait();
  const int j = blockIdx.x * gridDim.y + blockIdx.y;
  QImg Q{reinterpret_cast<uint2*>(img + (size_t)j * stride), reinterpret_cast<float2*>(img + (size_t)j * stride + gs_off)};
  if (is_h) {
    const float* h = reinterpret_cast<const float*>(src) + (size_t)j * n;
    qstage_vector([&](int j0, float (&v)[16]) { load_f32_16_cg(h + j0, v); }, n, G, Q, threadIdx.x, blockDim.x);
  } else {
    const uint16_t* x = reinterpret_cast<const uint16_t*>(src) + (size_t)j * n;
    qstage_vector([&](int j0, float (&v)[16]) { load_bf16_16(x + j0, v); }, n, G, Q, threadIdx.x, blockDim.x);
  }
  pdl_trigger();
}

// ---- the multi-token tile dot ---------------------------------------------

// NB bytes of code words from global memory, streaming (read once).
template <int NB>
__device__ __forceinline__ void ld_stream_words(const unsigned char* p, uint32_t* w) {
  if (NB >= 16) {
#pragma unroll
    for (int i = 0; i < NB / 16; ++i) {
      const uint4 v = ld_stream16(p + 16 * i);
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  } else if (NB == 8) {
    const uint2 v = ld_stream8(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
    w[0] = ld_stream4(p);
  }
}

// Blocks [0, nblk) of one tile in global memory against groups [g0, g0+nblk)
// of up to four tokens' images: col is the image whose B fragments this lane
// loads (token gid/2: the mma's column gid carries its hi or lo plane), tok
// the image of the lane's own token t (its group scales and sums). Lane
// (gid, t) accumulates token t: acc0 for local row gid, acc1 for row gid+8.
template <int BITS, int KS>
__device__ __forceinline__ void tile_dot_tokens(const unsigned char* blk0, int nblk, int g0, const unsigned char* col,
                                                const unsigned char* tok, int gs_off, float& acc0, float& acc1) {
  using F = TileFmt<BITS, KS>;
  constexpr int P = kGrpInFlight;
  const int lane = threadIdx.x & 31, gid = lane >> 2, t = lane & 3;
  // B fragments of column gid: token gid/2 (image col), plane hi (gid even) or lo
  const uint2* planes = reinterpret_cast<const uint2*>(col) + (gid & 1) * 4 + t;
  const float2* gs = reinterpret_cast<const float2*>(tok + gs_off);  // this lane's token
  for (int b0 = 0; b0 < nblk; b0 += P) {
    uint32_t w[P][F::NW];
    uint2 sb[P], bf[P][KS];
    float2 ms[P];
#pragma unroll
    for (int q = 0; q < P; ++q) {
      const int b = min(b0 + q, nblk - 1);
      const unsigned char* blk = blk0 + (size_t)b * F::BB;
      ld_stream_words<F::LB>(blk + lane * F::LB, w[q]);
      if (BITS == 3) ld_stream_words<F::LH>(blk + 32 * F::LB + lane * F::LH, w[q] + F::LB / 4);
      sb[q] = ld_stream8(blk + F::CB + gid * 8);
      const int g = g0 + b;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) bf[q][ks] = __ldcg(planes + (size_t)(g * KS + ks) * 8);
      ms[q] = __ldcg(gs + g);
    }
#pragma unroll
    for (int q = 0; q < P; ++q) {
      if (b0 + q >= nblk) continue;
      int d[4];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t a[4];
        extract_a<BITS, KS>(w[q], ks, a);
        mma_u8s8(d, a, bf[q][ks], ks > 0);
      }
      const float p0 = (float)(d[0] * 256 + d[1]) * ms[q].x;
      const float p1 = (float)(d[2] * 256 + d[3]) * ms[q].x;
      acc0 = fmaf(__uint_as_float(sb[q].x << 16), p0, acc0);
      acc0 = fmaf(__uint_as_float(sb[q].x & 0xFFFF0000u), ms[q].y, acc0);
      acc1 = fmaf(__uint_as_float(sb[q].y << 16), p1, acc1);
      acc1 = fmaf(__uint_as_float(sb[q].y & 0xFFFF0000u), ms[q].y, acc1);
    }
  }
}

// Token i of work item a: its (batch index, output slot). a < nsh is the
// shared expert (tokens a*kGrpMaxTok.., slot K); a >= nsh is chunk a-nsh of a
// routed expert, whose entries b*K + k sit in list from act[1] on.
__device__ __forceinline__ void unit_token(const GrpParams& p, int a, int i, int& b, int& k) {
  if (a < p.nsh) {
    b = a * kGrpSharedTok + i;
    k = p.f.K;
  } else {
    const int ent = p.g.list[p.g.act[3 * (a - p.nsh) + 1] + i];
    b = ent / p.f.K;
    k = ent % p.f.K;
  }
}

// ---- grouped gate/up and down -----------------------------------------------

// DOWN == false: gate/up tiles against x images, h per (token, slot).
// DOWN == true: down tiles against h images, y per (token, slot).
// FB, FKS: the one format (bits, k-steps per group) of every expert the
// instance serves when the routed and shared widths agree, so that only that
// tile dot is compiled in; FB == 0: any format, chosen per work item.
template <bool DOWN, int FB, int FKS>
__global__ void __launch_bounds__(kGrpWarps * 32, kGrpCtasPerSm) k_ffn_grp(GrpParams p) {
  constexpr int NP = DOWN ? kGrpPiecesDn : kGrpPiecesGu;  // warps per unit
  constexpr int NU = kGrpWarps / NP;                       // units per round
  __shared__ float part[NU][NP][kGrpMaxTok][kTileRows];
  __shared__ int s_tok[NU][kGrpMaxTok][2];
  const FfnParams& f = p.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  const int nunits = min(p.max_units, (p.nsh + p.g.nact[0]) * p.tps);
  const int u_end = nunits;
  // rounds of NU consecutive units, each CTA taking the next round
  // from the workspace counter when it is free: work items carry different
  // numbers of tokens (the shared expert's all of them), so a static deal
  // would leave the CTAs that drew the heavy units last; those come first in
  // the order and start first
  __shared__ int s_u0;
  int* next = p.g.nact + (DOWN ? 2 : 1);
  while (true) {
    if (threadIdx.x == 0) s_u0 = atomicAdd(next, NU);
    __syncthreads();
    const int u0 = s_u0;
    if (u0 >= nunits) break;
    // the units of this round and their token lists
    int ntok[NU];
#pragma unroll
    for (int r = 0; r < NU; ++r) {
      const int u = u0 + r;
      ntok[r] = 0;
      if (u < u_end) {
        const int a = u / p.tps;
        ntok[r] = a < p.nsh ? min(kGrpSharedTok, f.B - a * kGrpSharedTok) : p.g.act[3 * (a - p.nsh) + 2];
        for (int i = threadIdx.x; i < ntok[r]; i += blockDim.x) unit_token(p, a, i, s_tok[r][i][0], s_tok[r][i][1]);
      }
    }
    __syncthreads();
    const int r = warp / NP, q = warp % NP, u = u0 + r;
    if (u < u_end) {
      const int a = u / p.tps, T = u % p.tps;
      const bool routed = a >= p.nsh;
      const RecGeom& g = routed ? f.geo_r : f.geo_s;
      const uint8_t* rec = routed ? f.experts + (size_t)p.g.act[3 * (a - p.nsh)] * f.rec_r : f.shared;
      const int ng = DOWN ? (int)g.ng_i : (int)g.ng_h;
      const int g0 = q * ng / NP, g1 = (q + 1) * ng / NP;
      const unsigned char* blk =
          rec + (DOWN ? g.down_off + (size_t)T * g.D : (size_t)T * g.U) + (size_t)g0 * g.blk;
      for (int c0 = 0; c0 < ntok[r]; c0 += 4) {
        auto image = [&](int i) {
          i = min(c0 + i, ntok[r] - 1);
          const int src = DOWN ? s_tok[r][i][0] * (f.K + 1) + s_tok[r][i][1] : s_tok[r][i][0];
          return p.img + (size_t)src * p.img_stride;
        };
        const unsigned char* col = image(lane >> 3);  // token gid/2
        const unsigned char* tok = image(lane & 3);   // token t
        float acc0 = 0.f, acc1 = 0.f;
        auto dot = [&]<int BITS, int KS>() {
          tile_dot_tokens<BITS, KS>(blk, g1 - g0, g0, col, tok, p.img_gs_off, acc0, acc1);
        };
        if constexpr (FB == 0) with_fmt(routed ? f.bits_r : f.bits_s, f.G, dot);
        else dot.template operator()<FB, FKS>();
        const int i = c0 + (lane & 3);
        if (i < ntok[r]) {
          part[r][q][i][lane >> 2] = acc0;
          part[r][q][i][(lane >> 2) + 8] = acc1;
        }
      }
    }
    __syncthreads();
    // finish: gate/up -> h = silu(gate) * up for 8 units; down -> y rows
#pragma unroll
    for (int rr = 0; rr < NU; ++rr) {
      const int uu = u0 + rr;
      if (uu >= u_end) continue;
      const int T = uu % p.tps;
      const int per = DOWN ? kTileRows : 8;
      for (int j = threadIdx.x; j < ntok[rr] * per; j += blockDim.x) {
        const int i = j / per, row = j % per;
        const int b = s_tok[rr][i][0], k = s_tok[rr][i][1];
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int qq = 0; qq < NP; ++qq) {
          s0 += part[rr][qq][i][row];
          if (!DOWN) s1 += part[rr][qq][i][row + 8];
        }
        if (DOWN)
          f.y[((size_t)b * (f.K + 1) + k) * f.H + (size_t)T * kTileRows + row] = s0;
        else
          f.h[((size_t)b * (f.K + 1) + k) * f.I + 8 * T + row] = silu_f(s0) * s1;
      }
    }
    __syncthreads();
  }
  pdl_trigger();
}

}  // namespace moeq
