// stack.cuh -- moe_decode_layers: one token (batch 1) through n MoE layers in
// one persistent launch, one CTA per SM.
//
// Per layer l the whole grid runs, in the method's order (router logits ->
// softmax/top-K -> gate/up dequant mat-vecs + SwiGLU -> down dequant mat-vec
// -> combine with the shared expert and the residual -> RMSNorm for the next
// layer, as the Flash-MoE page lists its GPU kernels in "Metal Compute
// Shaders" and chains them in "Deferred GPU Expert Compute"):
//
//   stage x_l      every CTA: x_l = bf16(RMSNorm(r_l)) (l > 0) into shared
//                  memory, plus the fp16 image the dequant dots read
//   router         CTA c owns a contiguous range of router rows
//   sync 1         all logits written
//   top-K          the producer warp of every CTA selects the K experts
//   gate/up        CTA c owns a contiguous range of the shared expert's units
//                  and of the routed units (slot-major); h to global memory
//   sync 2         all of h written
//   down+combine   CTA c owns a contiguous range of 4-row output blocks: for
//                  every slot the rows' dot with h_k, weighted by the routing
//                  weight (shared: gamma), plus the residual
//   sync 3         r_{l+1} and its sum of squares complete
//
// Warp roles: warps 0..7 compute, warp 8 moves data. Because the record keeps
// a unit's gate/up rows and tables adjacent, and a CTA's ranges are
// contiguous, every weight byte the CTA needs arrives in few large bulk
// copies (cp.async.bulk, completion on mbarriers): ring items of up to four
// units or two router rows (about 16-18 KB), and one copy per slot of the
// CTA's down blocks into a region that fills as soon as the experts are
// known. A bulk copy's cost on this part is nearly fixed per copy below
// ~16 KB, so size, not count in flight, sets the rate. Router rows and
// shared-expert units of layer l+1 enter the ring while layer l finishes.
// Grid-wide syncs are monotonic arrival counters in the workspace (release
// reductions, acquire polls); every wait gives up after about a second, sets
// MOE_ERR_TIMEOUT and lets the kernel run to its end without further work.
#pragma once

#include "common.cuh"
#include "dqdot.cuh"
#include "router.cuh"

namespace moeq {

constexpr int kStackMaxLayers = 64;
constexpr int kCWarps = 8;                          // compute warps
constexpr int kCThreads = kCWarps * 32;
constexpr int kStackThreads = kCThreads + 32;       // + producer warp
constexpr int kDnBlk = kRowsPerDownBlock;           // rows per down block
constexpr int kMaxSlots = 16;
constexpr int kMaxRouterRowsPerCta = 8;
constexpr int kPiecesPerItem = 4;                   // units, or router half-rows, per ring item
constexpr int kMaxItems = 32;                       // ring items per layer per CTA
constexpr int kMaxPieces = kMaxItems * kPiecesPerItem;

enum { kItemRouter = 0, kItemGateUp = 1, kItemZero = 2 };

struct StackLayerPtrs {
  const uint8_t* experts;
  const uint8_t* shared;
  const uint16_t* router_w;
  const uint16_t* gate_w;
};

struct StackParams {
  StackLayerPtrs L[kStackMaxLayers];
  int n_layers;
  int H, I, E, K, G, bits_r, bits_s;
  unsigned long long rec_r;
  RecGeom geo_r, geo_s;
  const uint16_t* x_in;     // [H]
  const float* resid_in;    // [H] or null
  const int32_t* forced;    // [n_layers, K] or null
  int32_t* idx_out;         // [n_layers, K] or null
  float* w_out;             // [n_layers, K] or null
  float* resid_out;         // [H]
  uint16_t* xnorm_out;      // [H] or null
  float eps;
  int renorm;
  WsCtrl* ctrl;
  float* logits;            // [E]
  float* h;                 // [K+1, I]
  float* r;                 // [H]
  float* ss;                // [kStackMaxLayers]
  // shared-memory plan (byte offsets into the dynamic buffer)
  int sm_xs, sm_img4, sm_tab4, sm_inv4, sm_img2, sm_tab2, sm_inv2;
  int sm_himg, sm_htab, sm_hinv, himg_stride, htab_stride, hinv_stride;
  int sm_ring, slot_bytes, nslot, sm_regc, regc_slot_bytes;
  int need4, need2;
};

// CTA c's share [lo, hi) of n items split evenly over G CTAs.
__host__ __device__ inline int share_lo(int c, int G, int n) { return (int)((long long)n * c / G); }

// The static item plan of one CTA (identical for every layer): router items
// of up to two rows, shared-expert items of up to four units, routed items of
// up to four units that never straddle two slots.
struct ItemPlan {
  int n_items, n_router_items, n_pre;     // n_pre: router + shared items
  int n_pieces, n_router_pieces;
  int kind[kMaxItems];                    // kItemRouter or kItemGateUp
  int k[kMaxItems];                       // slot (routed), K (shared)
  int first[kMaxItems];                   // first router row / unit row of the item
  int npieces[kMaxItems];
  int piece0[kMaxItems];                  // index of the item's first piece
  int r0, nr;                             // router rows [r0, r0+nr)
  int b0, nblk;                           // down blocks [b0, b0+nblk)
};

__device__ void make_plan(const StackParams& p, ItemPlan& P) {
  const int c = blockIdx.x, G = gridDim.x;
  int n = 0, pc = 0;
  P.r0 = share_lo(c, G, p.E);
  P.nr = share_lo(c + 1, G, p.E) - P.r0;
  for (int r = 0; r < P.nr; r += 2) {
    P.kind[n] = kItemRouter;
    P.k[n] = 0;
    P.first[n] = r;
    P.npieces[n] = 2 * min(2, P.nr - r);
    P.piece0[n] = pc;
    pc += P.npieces[n];
    ++n;
  }
  P.n_router_items = n;
  P.n_router_pieces = pc;
  const int s0 = share_lo(c, G, p.I), s1 = share_lo(c + 1, G, p.I);
  for (int i = s0; i < s1; i += kPiecesPerItem) {
    P.kind[n] = kItemGateUp;
    P.k[n] = p.K;
    P.first[n] = i;
    P.npieces[n] = min(kPiecesPerItem, s1 - i);
    P.piece0[n] = pc;
    pc += P.npieces[n];
    ++n;
  }
  P.n_pre = n;
  const int u0 = share_lo(c, G, p.K * p.I), u1 = share_lo(c + 1, G, p.K * p.I);
  for (int u = u0; u < u1;) {
    const int k = u / p.I, i = u % p.I;
    const int cnt = min(kPiecesPerItem, min(u1 - u, p.I - i));
    P.kind[n] = kItemGateUp;
    P.k[n] = k;
    P.first[n] = i;
    P.npieces[n] = cnt;
    P.piece0[n] = pc;
    pc += cnt;
    ++n;
    u += cnt;
  }
  P.n_items = n;
  P.n_pieces = pc;
  P.b0 = share_lo(c, G, p.H / kDnBlk);
  P.nblk = share_lo(c + 1, G, p.H / kDnBlk) - P.b0;
}

// ---- producer pieces (lane 0 issues; the warp waits together) -------------

struct Ring {
  uint64_t* full;
  uint64_t* empty;
  int* last;     // per slot: item sequence number of the last fill issued (-1: none)
  unsigned char* base;
  int slot_bytes, nslot;
};

// Source and size of ring item `it` of layer l (0 bytes: an empty item,
// for a slot whose expert index was invalid).
__device__ __forceinline__ uint32_t item_source(const StackParams& p, const ItemPlan& P, int l, int it,
                                                const int* s_idx, const void** src) {
  if (P.kind[it] == kItemRouter) {
    *src = p.L[l].router_w + (size_t)(P.r0 + P.first[it]) * p.H;
    return (uint32_t)(P.npieces[it] / 2) * (uint32_t)p.H * 2;
  }
  if (P.k[it] == p.K) {
    *src = p.L[l].shared + (size_t)P.first[it] * p.geo_s.U;
    return (uint32_t)P.npieces[it] * p.geo_s.U;
  }
  const int e = s_idx[P.k[it]];
  if (e < 0) return 0u;
  *src = p.L[l].experts + (size_t)e * p.rec_r + (size_t)P.first[it] * p.geo_r.U;
  return (uint32_t)P.npieces[it] * p.geo_r.U;
}

// Issue ring items [it0, it1) of layer l, item it taking ring sequence number
// seq0 + (it - it0). The lanes issue in parallel: each round takes the run
// of next items whose slots are already free (lane j -> item next + j); if
// none is, lane 0 waits for the first. Returns false if a wait gave up.
__device__ bool issue_items(const StackParams& p, const ItemPlan& P, Ring& R, int l, int it0, int it1, uint32_t seq0,
                            const int* s_idx, const volatile int* abort) {
  const int lane = threadIdx.x & 31;
  const int width = min(32, R.nslot);
  for (int next = it0; next < it1;) {
    const int n = min(width, it1 - next);
    const uint32_t seq = seq0 + (uint32_t)(next - it0 + lane);
    const uint32_t slot = seq % R.nslot, fill = seq / R.nslot;
    const bool ready = lane < n && (fill == 0 || mbar_try_wait(&R.empty[slot], (fill - 1) & 1));
    int nr = __ffs(~__ballot_sync(0xFFFFFFFFu, ready)) - 1;  // ready run starting at lane 0
    if (nr < 0) nr = 32;
    nr = min(nr, n);
    if (nr == 0) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&R.empty[slot], (fill - 1) & 1, abort);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) return false;
      nr = 1;
    }
    if (lane < nr) {
      const void* src = nullptr;
      const uint32_t bytes = item_source(p, P, l, next + lane, s_idx, &src);
      R.last[slot] = (int)seq;
      mbar_arrive_expect_tx(&R.full[slot], bytes);
      if (bytes) bulk_g2s(R.base + (size_t)slot * R.slot_bytes, src, bytes, &R.full[slot]);
    }
    __syncwarp();
    next += nr;
  }
  return true;
}

// The CTA's down blocks of slots [k0, k1): one copy per slot (lane k - k0
// issues slot k's), all arming `bar`.
__device__ void issue_down(const StackParams& p, const ItemPlan& P, unsigned char* regc, int l, int k0, int k1,
                           const int* s_idx, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    uint32_t tot = 0;
    for (int k = k0; k < k1; ++k)
      if (k == p.K || s_idx[k] >= 0) tot += (uint32_t)P.nblk * (k == p.K ? p.geo_s.D : p.geo_r.D);
    mbar_arrive_expect_tx(bar, tot);
  }
  __syncwarp();
  const int k = k0 + lane;
  if (k < k1 && P.nblk > 0) {
    const bool shared = (k == p.K);
    if (shared || s_idx[k] >= 0) {
      const RecGeom& g = shared ? p.geo_s : p.geo_r;
      const uint8_t* rec = shared ? p.L[l].shared : p.L[l].experts + (size_t)s_idx[k] * p.rec_r;
      bulk_g2s(regc + (size_t)k * p.regc_slot_bytes, rec + g.down_off + (size_t)P.b0 * g.D, (uint32_t)P.nblk * g.D,
               bar);
    }
  }
  __syncwarp();
}

// Top-K (or forced picks) of layer l by the producer warp, from the logits
// every CTA published; registers only. Writes s_idx (-1 for an invalid pick)
// and s_w.
__device__ void producer_topk(const StackParams& p, int l, int* s_idx, float* s_w) {
  const int lane = threadIdx.x & 31;
  constexpr int MAXV = 32;  // E <= 1024
  float v[MAXV];
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < MAXV; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < p.E ? __ldcg(p.logits + e) : -INFINITY;
    mx = fmaxf(mx, v[j]);
  }
  mx = warp_max(mx);
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < MAXV; ++j) z += (lane + 32 * j < p.E) ? __expf(v[j] - mx) : 0.f;
  z = warp_sum(z);
  const int32_t* forced = p.forced ? p.forced + (size_t)l * p.K : nullptr;
  int pick_e = -1;     // lane k (< K) ends up holding pick k
  float pick_l = 0.f;  // and its logit
  for (int k = 0; k < p.K; ++k) {
    int bi;
    float best;
    if (forced) {
      bi = forced[k];
      const bool okf = bi >= 0 && bi < p.E;
      best = okf ? __ldcg(p.logits + bi) : -INFINITY;
      if (!okf) bi = -1;
    } else {
      best = -INFINITY;
      bi = 0x7FFFFFFF;
#pragma unroll
      for (int j = 0; j < MAXV; ++j) {
        const int e = lane + 32 * j;
        if (v[j] > best || (v[j] == best && e < bi)) {
          best = v[j];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, best, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (ov > best || (ov == best && oi < bi)) {
          best = ov;
          bi = oi;
        }
      }
      if (bi >= p.E || !(best > -INFINITY)) {
        bi = -1;  // no finite logit left (NaN input): no expert
      } else {
#pragma unroll
        for (int j = 0; j < MAXV; ++j)  // remove the pick from its owner lane
          if (lane + 32 * j == bi) v[j] = -INFINITY;
      }
    }
    if (lane == k) {
      pick_e = bi;
      pick_l = best;
    }
  }
  if (lane < p.K && pick_e < 0) set_error(p.ctrl, MOE_ERR_INDEX);
  float pw = (lane < p.K && pick_e >= 0) ? __expf(pick_l - mx) / z : 0.f;
  float tot = pw;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xFFFFFFFFu, tot, o);
  if (lane < p.K) {
    const float wk = (p.renorm && tot > 0.f) ? pw / tot : pw;
    s_idx[lane] = pick_e;
    s_w[lane] = wk;
    if (blockIdx.x == 0) {
      if (p.idx_out) p.idx_out[(size_t)l * p.K + lane] = forced ? forced[lane] : pick_e;
      if (p.w_out) p.w_out[(size_t)l * p.K + lane] = wk;
    }
  }
  __syncwarp();
}

// ---- compute pieces ------------------------------------------------------------

// Gate and up rows of one unit from a ring slot; returns h in lane 0.
template <int BITS>
__device__ __forceinline__ float gateup_from_slot(const unsigned char* slot, int H, int G, const ImgRef& R) {
  const int lane = threadIdx.x & 31;
  const int rowb = H * BITS / 8, ng = H / G, nchunk = H * BITS / 128;
  const bool two = (BITS == 2) && (G == 32);
  const uint32_t* gsb = reinterpret_cast<const uint32_t*>(slot + 2 * rowb);
  const uint32_t* usb = gsb + ng;
  float part[2] = {0.f, 0.f};
  for (int c = lane; c < nchunk; c += 32) {
    const uint4 qg = *reinterpret_cast<const uint4*>(slot + (size_t)c * 16);
    const uint4 qu = *reinterpret_cast<const uint4*>(slot + rowb + (size_t)c * 16);
    const int g = chunk_group<BITS>(c, G, two);
    const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, R);
    part[0] += chunk_dot_x<BITS>(qg, X, gsb[g], two ? gsb[g + 1] : 0u, two);
    part[1] += chunk_dot_x<BITS>(qu, X, usb[g], two ? usb[g + 1] : 0u, two);
  }
  const float v = transpose_reduce<2>(part);
  const float up = __shfl_sync(0xFFFFFFFFu, v, 16);
  return silu_f(v) * up;
}

// Adds coef * (4 rows of one down block) into acc (per-lane partials).
template <int BITS>
__device__ __forceinline__ void down_block_acc(const unsigned char* blk, int I, int G, const ImgRef& R, float coef,
                                               float (&acc)[kDnBlk]) {
  const int lane = threadIdx.x & 31;
  const int rowb = I * BITS / 8, ng = I / G, nchunk = I * BITS / 128;
  const bool two = (BITS == 2) && (G == 32);
  const uint32_t* sb = reinterpret_cast<const uint32_t*>(blk + kDnBlk * rowb);
  for (int c = lane; c < nchunk; c += 32) {
    const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, R);
    const int g = chunk_group<BITS>(c, G, two);
#pragma unroll
    for (int r = 0; r < kDnBlk; ++r) {
      const uint4 q = *reinterpret_cast<const uint4*>(blk + (size_t)r * rowb + (size_t)c * 16);
      acc[r] += coef * chunk_dot_x<BITS>(q, X, sb[r * ng + g], two ? sb[r * ng + g + 1] : 0u, two);
    }
  }
}

__device__ __forceinline__ ImgRef stack_img(unsigned char* sm, int img, int tab, int inv) {
  return ImgRef{reinterpret_cast<uint4*>(sm + img), reinterpret_cast<float4*>(sm + tab),
                reinterpret_cast<float*>(sm + inv)};
}

__device__ __forceinline__ ImgRef stack_himg(unsigned char* sm, const StackParams& p, int k) {
  return ImgRef{reinterpret_cast<uint4*>(sm + p.sm_himg + (size_t)k * p.himg_stride),
                reinterpret_cast<float4*>(sm + p.sm_htab + (size_t)k * p.htab_stride),
                reinterpret_cast<float*>(sm + p.sm_hinv + (size_t)k * p.hinv_stride)};
}

// Stage x_l, 16 inputs per thread: read the inputs (x_in for layer 0, else
// bf16(r * inv_norm)), write the bf16 copy the router reads and the image of
// the primary width; returns the thread's partial dot with the shared-gate
// vector.
template <int BITS>
__device__ __forceinline__ float stage_x_primary(const StackParams& p, int l, float inv_norm, uint16_t* xs, ImgRef R,
                                                 const uint16_t* gw, int tid) {
  float gdot = 0.f;
  auto get = [&](int j0, float (&v)[16]) {
    if (l == 0) {
      load_bf16_16(p.x_in + j0, v);
    } else {
      load_f32_16_cg(p.r + j0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = bf16_bits_to_f32(f32_to_bf16_bits(v[j] * inv_norm));
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        w[i] = (__float_as_uint(v[8 * q + 2 * i]) >> 16) | (__float_as_uint(v[8 * q + 2 * i + 1]) & 0xFFFF0000u);
      reinterpret_cast<uint4*>(xs + j0)[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (gw) {
      float g[16];
      load_bf16_16(gw + j0, g);
#pragma unroll
      for (int j = 0; j < 16; ++j) gdot += g[j] * v[j];
    }
  };
  for (int gi = tid >> 5; gi * 32 < p.H / 16; gi += kCWarps) stage_group<BITS>(get, p.H, R, gi, tid & 31);
  return gdot;
}

// A second image width staged from the bf16 copy in shared memory.
template <int BITS>
__device__ __forceinline__ void stage_x_secondary(int H, const uint16_t* xs, ImgRef R, int tid) {
  stage_vector<BITS>([&](int j0, float (&v)[16]) { load_bf16_16(xs + j0, v); }, H, R, tid, kCThreads);
}

// Stage h ([K+1, I] fp32 in the workspace): warp job = (slot, 32 segments).
__device__ __forceinline__ void stage_h_stack(const StackParams& p, unsigned char* sm, int tid) {
  const int I = p.I, K = p.K;
  const int jobs_per_slot = (I / 16 + 31) / 32;
  for (int j = tid >> 5; j < (K + 1) * jobs_per_slot; j += kCWarps) {
    const int k = j / jobs_per_slot, gi = j % jobs_per_slot;
    const float* hk = p.h + (size_t)k * I;
    const ImgRef R = stack_himg(sm, p, k);
    auto get = [&](int j0, float (&v)[16]) { load_f32_16_cg(hk + j0, v); };
    if ((k < K ? p.bits_r : p.bits_s) == 4)
      stage_group<4>(get, I, R, gi, tid & 31);
    else
      stage_group<2>(get, I, R, gi, tid & 31);
  }
}


__global__ void __launch_bounds__(kStackThreads, 1) k_decode_layers(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t full_bar[kMaxSlots], empty_bar[kMaxSlots], c_bar[2], cfree_bar;
  __shared__ int s_last[kMaxSlots];
  __shared__ int s_idx[MOEQ_MAX_K];
  __shared__ float s_w[MOEQ_MAX_K];
  __shared__ float s_part[kMaxRouterRowsPerCta][2];
  __shared__ float s_misc[4];  // 1: shared-gate dot; 2: CTA sum of squares
  __shared__ unsigned char s_piece_item[kMaxPieces];
  __shared__ ItemPlan P;
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  unsigned* sync_count = &p.ctrl->sync_count;

  if (tid == 0) {
    make_plan(p, P);
    for (int it = 0; it < P.n_items; ++it)
      for (int q = 0; q < P.npieces[it]; ++q) s_piece_item[P.piece0[it] + q] = (unsigned char)it;
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kPiecesPerItem);
      s_last[i] = -1;
    }
    mbar_init(&c_bar[0], 1);
    mbar_init(&c_bar[1], 1);
    mbar_init(&cfree_bar, kCWarps);
    s_abort = 0;
    s_misc[1] = 0.f;
    s_misc[2] = 0.f;
    fence_mbar_init();
  }
  __syncthreads();

  auto fail = [&](void) {
    set_error(p.ctrl, MOE_ERR_TIMEOUT);
    s_abort = 1;
  };
  const int n_items = P.n_items;

  if (warp == kCWarps) {
    // ===================== producer warp =====================
    Ring R{full_bar, empty_bar, s_last, sm + p.sm_ring, p.slot_bytes, p.nslot};
    unsigned char* regc = sm + p.sm_regc;
    int c_last[2] = {-1, -1};  // last layer whose down copies were issued, per down barrier
    if (!issue_items(p, P, R, 0, 0, P.n_pre, 0u, s_idx, &s_abort) && lane == 0) fail();
    for (int l = 0; l < p.n_layers; ++l) {
      if (l > 0 && !mbar_wait(&cfree_bar, (l - 1) & 1, &s_abort) && lane == 0) fail();
      __syncwarp();
      // shared expert's down blocks (known before routing)
      if (!s_abort) {
        issue_down(p, P, regc, l, p.K, p.K + 1, s_idx, &c_bar[0]);
        c_last[0] = l;
      }
      // routing
      if (!counter_wait(sync_count, (unsigned)(3 * l + 1) * G, &s_abort) && lane == 0) fail();
      __syncwarp();
      producer_topk(p, l, s_idx, s_w);
      // routed gate/up units (first as many as the ring takes now), the
      // routed down blocks, then the remaining units
      const uint32_t seq_l = (uint32_t)(l * n_items);
      const int first = min(n_items, P.n_pre + p.nslot);
      bool ok = issue_items(p, P, R, l, P.n_pre, first, seq_l + P.n_pre, s_idx, &s_abort);
      if (!s_abort) {
        issue_down(p, P, regc, l, 0, p.K, s_idx, &c_bar[1]);
        c_last[1] = l;
      }
      if (ok) ok = issue_items(p, P, R, l, first, n_items, seq_l + first, s_idx, &s_abort);
      if (ok && l + 1 < p.n_layers)
        ok = issue_items(p, P, R, l + 1, 0, P.n_pre, (uint32_t)((l + 1) * n_items), s_idx, &s_abort);
      if (!ok && lane == 0 && !s_abort) fail();
      __syncwarp();
    }
    // drain: every copy issued must have landed before the CTA exits
    if (lane == 0) {
      for (int slot = 0; slot < p.nslot; ++slot) {
        const int j = s_last[slot];
        if (j < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(&full_bar[slot], (j / p.nslot) & 1) && clock64() - t0 < kWaitBudgetCycles) {
        }
      }
      for (int q = 0; q < 2; ++q) {
        if (c_last[q] < 0) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(&c_bar[q], c_last[q] & 1) && clock64() - t0 < kWaitBudgetCycles) {
        }
      }
    }
    __syncwarp();
  } else {
    // ===================== compute warps =====================
    const int H = p.H, I = p.I, K = p.K;
    uint16_t* xs = reinterpret_cast<uint16_t*>(sm + p.sm_xs);
    const ImgRef X4 = stack_img(sm, p.sm_img4, p.sm_tab4, p.sm_inv4);
    const ImgRef X2 = stack_img(sm, p.sm_img2, p.sm_tab2, p.sm_inv2);
    const unsigned char* ring = sm + p.sm_ring;
    const unsigned char* regc = sm + p.sm_regc;
    const int n_pieces = P.n_pieces, n_rp = P.n_router_pieces;

    for (int l = 0; l < p.n_layers; ++l) {
      // ---- stage x_l ----
      float inv_norm = 1.f;
      if (l > 0) {
        if (tid == 0 && !counter_wait(sync_count, (unsigned)(3 * l) * G, &s_abort)) fail();
        named_sync(1, kCThreads);
        inv_norm = rsqrtf(__ldcg(p.ss + (l - 1)) / (float)H + p.eps);
      }
      const uint16_t* gw = p.L[l].gate_w;
      const float gdot = p.need4 ? stage_x_primary<4>(p, l, inv_norm, xs, X4, gw, tid)
                                 : stage_x_primary<2>(p, l, inv_norm, xs, X2, gw, tid);
      if (gw) {
        const float d = warp_sum(gdot);
        if (lane == 0) atomicAdd(&s_misc[1], d);
      }
      named_sync(1, kCThreads);
      if (p.need4 && p.need2) {
        stage_x_secondary<2>(H, xs, X2, tid);
        named_sync(1, kCThreads);
      }
      const float gamma = gw ? 1.f / (1.f + expf(-s_misc[1])) : 1.f;

      // ---- ring pieces: router half-rows, then gate/up units ----
      bool router_synced = false;
      auto router_barrier = [&](void) {
        if (warp == 0) {
          named_sync(2, kCThreads);
          if (lane == 0) {
            for (int m = 0; m < P.nr; ++m) __stcg(p.logits + P.r0 + m, s_part[m][0] + s_part[m][1]);
            arrive_release_gpu(sync_count);
          }
          __syncwarp();
        } else {
          named_arrive(2, kCThreads);
        }
      };
      for (int pc = warp; pc < n_pieces; pc += kCWarps) {
        if (!router_synced && pc >= n_rp) {
          router_barrier();
          router_synced = true;
        }
        const int it = s_piece_item[pc];
        const int pos = pc - P.piece0[it];
        const uint32_t seq = (uint32_t)(l * n_items + it);
        const int slot = seq % p.nslot;
        const bool ok = mbar_wait(&full_bar[slot], (seq / p.nslot) & 1, &s_abort);
        if (!ok && lane == 0 && !s_abort) fail();
        if (ok) {
          const unsigned char* sl = ring + (size_t)slot * p.slot_bytes;
          if (P.kind[it] == kItemRouter) {
            const int row = pos >> 1, half = pos & 1;
            const int nv = H / 16;  // 16-byte words in a half row
            const uint4* wv = reinterpret_cast<const uint4*>(sl + (size_t)row * H * 2 + (size_t)half * H);
            const uint4* xv = reinterpret_cast<const uint4*>(xs + half * (H / 2));
            float acc = 0.f;
            for (int v = lane; v < nv; v += 32) acc = dot8_bf16(wv[v], xv[v], acc);
            acc = warp_sum(acc);
            if (lane == 0) s_part[P.first[it] + row][half] = acc;
          } else {
            const int k = P.k[it], i = P.first[it] + pos;
            const bool routed = k < K;
            float hv = 0.f;
            if (!routed || s_idx[k] >= 0) {
              const int bits = routed ? p.bits_r : p.bits_s;
              const RecGeom& g = routed ? p.geo_r : p.geo_s;
              const unsigned char* unit = sl + (size_t)pos * g.U;
              hv = bits == 4 ? gateup_from_slot<4>(unit, H, p.G, X4) : gateup_from_slot<2>(unit, H, p.G, X2);
            }
            if (lane == 0) __stcg(p.h + (size_t)k * I + i, hv);
          }
        }
        __syncwarp();
        if (lane == 0) {
          const uint32_t cnt = (pos == 0) ? (uint32_t)(kPiecesPerItem - P.npieces[it] + 1) : 1u;
          mbar_arrive_cnt(&empty_bar[slot], cnt);
        }
      }
      if (!router_synced) router_barrier();

      // ---- sync 2: h complete ----
      named_sync(1, kCThreads);
      if (tid == 0) {
        arrive_release_gpu(sync_count);
        if (!counter_wait(sync_count, (unsigned)(3 * l + 2) * G, &s_abort)) fail();
      }
      named_sync(1, kCThreads);

      // ---- stage h images (one per slot) ----
      if (tid == 0) s_misc[1] = 0.f;  // gate dot of the next layer starts from zero
      stage_h_stack(p, sm, tid);
      named_sync(1, kCThreads);

      // ---- down + combine for this CTA's row blocks ----
      const bool ok0 = mbar_wait(&c_bar[0], l & 1, &s_abort);
      const bool ok1 = mbar_wait(&c_bar[1], l & 1, &s_abort);
      if (!(ok0 && ok1) && tid == 0 && !s_abort) fail();
      float ssq = 0.f;
      for (int m = warp; m < P.nblk; m += kCWarps) {
        const int i0 = (P.b0 + m) * kDnBlk;
        float acc[kDnBlk] = {0.f, 0.f, 0.f, 0.f};
        if (!s_abort) {
          for (int k = 0; k <= K; ++k) {
            // s_idx/s_w were written before the routed down copies were armed
            const float wk = k < K ? (s_idx[k] >= 0 ? s_w[k] : 0.f) : gamma;
            if (wk == 0.f) continue;
            const RecGeom& g = k < K ? p.geo_r : p.geo_s;
            const unsigned char* blk = regc + (size_t)k * p.regc_slot_bytes + (size_t)m * g.D;
            const ImgRef R = stack_himg(sm, p, k);
            if ((k < K ? p.bits_r : p.bits_s) == 4)
              down_block_acc<4>(blk, I, p.G, R, wk, acc);
            else
              down_block_acc<2>(blk, I, p.G, R, wk, acc);
          }
        }
        const float tot = transpose_reduce<kDnBlk>(acc);
        if ((lane & 7) == 0) {
          const int i = i0 + (lane >> 3);
          float r0;
          if (l == 0)
            r0 = p.resid_in ? p.resid_in[i] : bf16_bits_to_f32(p.x_in[i]);
          else
            r0 = __ldcg(p.r + i);
          const float out = r0 + tot;
          if (l + 1 < p.n_layers)
            __stcg(p.r + i, out);
          else
            p.resid_out[i] = out;
          ssq += out * out;
        }
      }
      ssq = warp_sum(ssq);
      if (lane == 0) {
        atomicAdd(&s_misc[2], ssq);
        mbar_arrive(&cfree_bar);
      }
      // ---- sync 3: r_{l+1} complete ----
      named_sync(1, kCThreads);
      if (tid == 0) {
        atomicAdd(p.ss + l, s_misc[2]);
        s_misc[2] = 0.f;
        arrive_release_gpu(sync_count);
      }
    }

    // ---- optional RMSNorm'd bf16 output of the last layer ----
    if (p.xnorm_out) {
      if (tid == 0 && !counter_wait(sync_count, (unsigned)(3 * p.n_layers) * G, &s_abort)) fail();
      named_sync(1, kCThreads);
      const float inv = rsqrtf(__ldcg(p.ss + (p.n_layers - 1)) / (float)H + p.eps);
      for (int t = tid; t < P.nblk * kDnBlk; t += kCThreads) {
        const int i = P.b0 * kDnBlk + t;
        p.xnorm_out[i] = f32_to_bf16_bits(__ldcg(p.resid_out + i) * inv);
      }
    }
  }

  // ---- leave: the last CTA out resets the grid counters ----
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&p.ctrl->exit_count, 1u);
    if (t == (unsigned)G - 1) {
      atomicExch(&p.ctrl->sync_count, 0u);
      for (int l = 0; l < p.n_layers; ++l) p.ss[l] = 0.f;
      __threadfence();
      atomicExch(&p.ctrl->exit_count, 0u);
    }
  }
}

}  // namespace moeq
