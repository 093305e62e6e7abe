// grouped.cuh -- moe_expert_ffn_q for a batch of tokens, grouped by expert:
// each active expert's weights are read once per step for all the tokens
// routed to it (the batched-decode token grouping; the pages themselves run
// one token at a time).
//
//   k_group           stable counting sort of the (token, slot) picks by
//                     expert id: cnt, off, list, and the work items (an
//                     expert's entries in chunks of at most kGrpMaxTok)
//   k_stage_batch     the input image of every token (x, or h per slot) in
//                     the workspace, so that a tile can be applied to
//                     several tokens without restaging
//   k_ffn_grp<DOWN>   unit = (work item, tile). One CTA per SM: a copy warp
//                     streams the CTA's units' tiles with bulk copies into a
//                     ring of shared-memory slots; each compute warp takes a
//                     piece = (unit, four of its tokens) and runs the whole
//                     tile against those four tokens' images (four tokens
//                     share each mma: columns 2t, 2t+1 carry token t's hi and
//                     lo planes), so a lane ends with finished outputs and no
//                     partial sums cross warps. gate/up: h per (token, slot);
//                     down: y per (token, slot).
//
// The work items of a step are [shared expert (every token, slot K),
// routed chunks by expert id].
#pragma once

#include "common.cuh"
#include "ffn.cuh"
#include "tiledot.cuh"

namespace moeq {

constexpr int kGrpWarps = 15;                         // compute warps (one more copies tiles: 16 warps, 128 registers)
constexpr int kGrpThreads = (kGrpWarps + 1) * 32;
constexpr int kGrpMaxTok = 128;                       // entries of one work item at most
constexpr int kGrpMaxPieces = kGrpMaxTok / 4;         // pieces of one unit at most
constexpr int kGrpMaxSlots = 16;                      // ring slots
static_assert(MOEQ_MAX_B <= kGrpMaxTok, "the shared expert's tokens are one work item");

// A routed expert with more than kGrpMaxTok entries (forced picks may repeat
// an expert within a token) is split into several chunks; a chunk is one
// work item.
constexpr int kGrpExtraChunks = (MOEQ_MAX_B * MOEQ_MAX_K) / kGrpMaxTok;
struct GrpWs {
  int* cnt;   // [E]
  int* off;   // [E + 1]
  int* list;  // [B*K]: entries b*K + k grouped by expert, in entry order
  int* act;   // [E + kGrpExtraChunks][3]: (expert, its first entry in list, entries) per chunk, by expert id
  int* nact;  // [1]: chunks
};

struct GrpParams {
  FfnParams f;
  GrpWs g;
  unsigned char* img;   // per-source images: x [B] (gate/up) or h [B][K+1] (down)
  int img_stride;       // bytes between consecutive images
  int img_gs_off;       // byte offset of the gs array within an image
  int tps;              // tiles per expert (I/8 gate/up, H/16 down)
  int max_units;        // (1 + most work items) * tps
  int slot_bytes, nslot;  // ring of tile slots in dynamic shared memory
};

// ---- grouping -------------------------------------------------------------

// One CTA. Picks outside [0, E) set MOE_ERR_INDEX, are left out of every
// group, and get a zero output slot here.
__global__ void __launch_bounds__(256) k_group(const int32_t* idx, int B, int K, int E, int H, GrpWs g, float* y,
                                               WsCtrl* ctrl) {
  extern __shared__ int s_cnt[];  // [E + 1]
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
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = idx[i];
    if (e < 0 || e >= E) continue;
    int r = 0;
    for (int j = 0; j < i; ++j) r += idx[j] == e;
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

// One whole tile in shared memory (nblk blocks) against four tokens' images
// in global memory (imgs[c]; the lanes of column pair c read image c). Lane
// (gid, t) accumulates token t: acc0 for local row gid, acc1 for row gid+8.
// The images' fragments of the next P groups are loaded ahead (they come
// from L2).
template <int BITS, int KS>
__device__ __forceinline__ void tile_dot_tokens(const unsigned char* tile, int nblk,
                                                const unsigned char* const (&imgs)[4], int gs_off, float& acc0,
                                                float& acc1) {
  using F = TileFmt<BITS, KS>;
  constexpr int P = KS >= 4 ? 4 : 8;  // groups in flight (about 16 KB of fragments per warp)
  const int lane = threadIdx.x & 31, gid = lane >> 2, t = lane & 3;
  // B fragments of column gid: token gid/2, plane hi (gid even) or lo
  const uint2* planes = reinterpret_cast<const uint2*>(imgs[gid >> 1]) + (gid & 1) * 4 + t;
  const float2* gs = reinterpret_cast<const float2*>(imgs[t] + gs_off);  // this lane's token
  uint2 bf[P][KS];
  float2 ms[P];
#pragma unroll
  for (int q = 0; q < P; ++q) {
    const int g = min(q, nblk - 1);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) bf[q][ks] = __ldg(planes + (size_t)(g * KS + ks) * 8);
    ms[q] = __ldg(gs + g);
  }
  for (int b0 = 0; b0 < nblk; b0 += P) {
#pragma unroll
    for (int q = 0; q < P; ++q) {
      const int b = b0 + q;
      if (b < nblk) {
        const unsigned char* blk = tile + (size_t)b * F::BB;
        uint32_t w[F::NW];
        load_lane_codes<BITS, KS>(blk, lane, w);
        const uint2 sb = *reinterpret_cast<const uint2*>(blk + F::CB + gid * 8);
        int d[4];
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t a[4];
          extract_a<BITS, KS>(w, ks, a);
          mma_u8s8(d, a, bf[q][ks], ks > 0);
        }
        const float p0 = (float)(d[0] * 256 + d[1]) * ms[q].x;
        const float p1 = (float)(d[2] * 256 + d[3]) * ms[q].x;
        acc0 = fmaf(__uint_as_float(sb.x << 16), p0, acc0);
        acc0 = fmaf(__uint_as_float(sb.x & 0xFFFF0000u), ms[q].y, acc0);
        acc1 = fmaf(__uint_as_float(sb.y << 16), p1, acc1);
        acc1 = fmaf(__uint_as_float(sb.y & 0xFFFF0000u), ms[q].y, acc1);
        const int nb = b + P;
        if (nb < nblk) {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) bf[q][ks] = __ldg(planes + (size_t)(nb * KS + ks) * 8);
          ms[q] = __ldg(gs + nb);
        }
      }
    }
  }
}

// A work item's tokens: (batch index, output slot) of its i-th entry. Work
// item 0 is the shared expert (every token, slot K); work item a >= 1 is
// chunk a-1 of a routed expert, whose entries b*K + k sit in list from
// `start` on.
struct GrpItem {
  int a, ntok, start;
};
__device__ __forceinline__ GrpItem grp_item(const GrpParams& p, int a) {
  if (a == 0) return GrpItem{0, p.f.B, 0};
  const int* c = p.g.act + 3 * (a - 1);
  return GrpItem{a, c[2], c[1]};
}
__device__ __forceinline__ int2 item_token(const GrpParams& p, const GrpItem& it, int i) {
  if (it.a == 0) return make_int2(i, p.f.K);
  const int ent = __ldg(p.g.list + it.start + i);
  return make_int2(ent / p.f.K, ent % p.f.K);
}

// ---- grouped gate/up and down -----------------------------------------------

// DOWN == false: gate/up tiles against x images, h per (token, slot).
// DOWN == true: down tiles against h images, y per (token, slot).
// CTA c takes a contiguous share of the step's units; its copy warp fills the
// ring in unit order and its compute warps take the units' pieces in turn
// (piece j of the CTA's sequence goes to warp j % kGrpWarps). A slot is free
// once every piece of its unit has arrived on its empty barrier (the first
// piece arrives for the pieces the unit does not have). Every wait is
// bounded: on a timeout the CTA records MOE_ERR_TIMEOUT, skips the rest of
// its work and waits (bounded) for its copies in flight before it leaves.
template <bool DOWN>
__global__ void __launch_bounds__(kGrpThreads, 1) k_ffn_grp(const __grid_constant__ GrpParams p) {
  extern __shared__ __align__(128) unsigned char ring[];
  __shared__ __align__(8) uint64_t full_bar[kGrpMaxSlots], empty_bar[kGrpMaxSlots];
  __shared__ int s_last[kGrpMaxSlots];
  __shared__ volatile int s_abort;
  const FfnParams& f = p.f;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kGrpMaxPieces);
      s_last[i] = -1;
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();
  const long long budget = wait_budget(f.ctrl);
  const int nunits = min(p.max_units, (1 + p.g.nact[0]) * p.tps);
  const int u_lo = (int)((long long)nunits * blockIdx.x / gridDim.x);
  const int u_hi = (int)((long long)nunits * (blockIdx.x + 1) / gridDim.x);
  auto unit_rec = [&](int a, const RecGeom*& g) -> const uint8_t* {
    g = a == 0 ? &f.geo_s : &f.geo_r;
    return a == 0 ? f.shared : f.experts + (size_t)p.g.act[3 * (a - 1)] * f.rec_r;
  };

  if (warp == kGrpWarps) {
    // ---- copy warp: one tile per unit into the ring, in unit order ----
    for (int u = u_lo; u < u_hi && !s_abort; ++u) {
      const int seq = u - u_lo, slot = seq % p.nslot, fill = seq / p.nslot;
      bool ok = true;
      if (lane == 0) {
        if (fill > 0) ok = mbar_wait(&empty_bar[slot], (uint32_t)((fill - 1) & 1), &s_abort, budget);
        if (ok) {
          const int a = u / p.tps, T = u % p.tps;
          const RecGeom* g;
          const uint8_t* rec = unit_rec(a, g);
          const uint8_t* src = rec + (DOWN ? g->down_off + (size_t)T * g->D : (size_t)T * g->U);
          const uint32_t bytes = DOWN ? g->D : g->U;
          *reinterpret_cast<volatile int*>(&s_last[slot]) = seq;
          mbar_arrive_expect_tx(&full_bar[slot], bytes);
          bulk_g2s(ring + (size_t)slot * p.slot_bytes, src, bytes, &full_bar[slot]);
        } else if (!s_abort) {
          set_error(f.ctrl, MOE_ERR_TIMEOUT);
          s_abort = 1;
        }
      }
      __syncwarp();
    }
    // every copy issued must land before the CTA leaves (bounded)
    if (lane < p.nslot) {
      const int j = s_last[lane];
      if (j >= 0) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&full_bar[lane], (uint32_t)((j / p.nslot) & 1)) && clock64() - t0 < budget) {
        }
      }
    }
  } else {
    // ---- compute warps: pieces (unit, four tokens) in turn ----
    int pc = 0;  // pieces of the CTA's units before unit u
    GrpItem it{-1, 0, 0};
    for (int u = u_lo; u < u_hi; ++u) {
      const int a = u / p.tps, T = u % p.tps;
      if (a != it.a) it = grp_item(p, a);  // a work item spans tps consecutive units
      const int np = (it.ntok + 3) / 4;
      const int first = (warp - pc % kGrpWarps + kGrpWarps) % kGrpWarps;  // this warp's first piece of the unit
      const int seq = u - u_lo, slot = seq % p.nslot;
      for (int c = first; c < np; c += kGrpWarps) {
        // the four tokens' (batch index, slot): one L2 round trip, issued
        // before the wait for the tile
        int2 tok[4];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tok[cc] = item_token(p, it, min(4 * c + cc, it.ntok - 1));
        // wait until the copy warp has issued this fill, then for its bytes
        bool ok = true;
        if (lane == 0) {
          const volatile int* last = s_last;
          const long long t0 = clock64();
          while (last[slot] != seq) {
            if (s_abort || clock64() - t0 > budget) {
              ok = false;
              break;
            }
            __nanosleep(64);
          }
          ok = ok && mbar_wait(&full_bar[slot], (uint32_t)((seq / p.nslot) & 1), &s_abort, budget);
          if (!ok && !s_abort) {
            set_error(f.ctrl, MOE_ERR_TIMEOUT);
            s_abort = 1;
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          const unsigned char* imgs[4];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            imgs[cc] = p.img + (size_t)(DOWN ? tok[cc].x * (f.K + 1) + tok[cc].y : tok[cc].x) * p.img_stride;
          const RecGeom* g;
          unit_rec(a, g);
          const bool routed = a != 0;
          const int nblk = DOWN ? (int)g->ng_i : (int)g->ng_h;
          float acc0 = 0.f, acc1 = 0.f;
          with_fmt(routed ? f.bits_r : f.bits_s, f.G, [&]<int BITS, int KS>() {
            tile_dot_tokens<BITS, KS>(ring + (size_t)slot * p.slot_bytes, nblk, imgs, p.img_gs_off, acc0, acc1);
          });
          const int cc = lane & 3;
          if (4 * c + cc < it.ntok) {
            const int2 tk = cc == 0 ? tok[0] : (cc == 1 ? tok[1] : (cc == 2 ? tok[2] : tok[3]));
            const int b = tk.x, k = tk.y, gid = lane >> 2;
            if (DOWN) {
              float* y = f.y + ((size_t)b * (f.K + 1) + k) * f.H + (size_t)T * kTileRows;
              y[gid] = acc0;
              y[gid + 8] = acc1;
            } else {
              f.h[((size_t)b * (f.K + 1) + k) * f.I + 8 * T + gid] = silu_f(acc0) * acc1;
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(&empty_bar[slot], c == 0 ? (uint32_t)(kGrpMaxPieces - np + 1) : 1u);
      }
      pc += np;
    }
  }
  pdl_trigger();
}

}  // namespace moeq
