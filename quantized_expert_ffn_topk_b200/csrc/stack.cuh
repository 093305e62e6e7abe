// stack.cuh -- moe_decode_layers: one token (batch 1) through n MoE layers in
// one persistent launch, one CTA per SM.
//
// Per layer l the grid runs the method's steps in order (router logits ->
// softmax/top-K -> gate/up dequant mat-vecs + SwiGLU -> down dequant mat-vec
// -> combine with the shared expert and the residual -> RMSNorm for the next
// layer, as the Flash-MoE page lists its GPU kernels in "Metal Compute
// Shaders" and chains them in "Deferred GPU Expert Compute"):
//
//   stage x_l     every CTA reads r_l (all of it), forms its sum of squares
//                 itself, and stages x_l = bf16(RMSNorm(r_l)) (layer 0: the
//                 input) as a bf16 copy for the router and an image for the
//                 tensor-core dots
//   router        CTA c owns a contiguous range of router rows
//   top-K         the compute warps of every CTA select from all logits
//   shared expert gate/up tiles before the routing is known, then its down
//                 tiles as soon as every CTA's shared h is out
//   routed        gate/up tiles (slot-major ranges), then down tiles
//   combine       CTA c owns a contiguous range of 16-row output tiles: the
//                 routing-weighted slot sums plus the residual give r_{l+1}
//
// Data crosses CTAs through the workspace (logits, h, r at L2), published by
// monotonic arrival counters: each CTA adds one (release) when its part is
// out, and one thread per reading CTA polls (acquire) before the CTA reads.
//
// Warp roles: warps 0..15 compute, warp 16 moves data with bulk copies
// (cp.async.bulk, completion on mbarriers) into a ring of slots: router items
// (two rows), gate/up items (half a tile) and down items (the CTA's down
// tiles of one slot). Router rows and shared-expert tiles of layer l+1 enter
// the ring while layer l finishes. Every wait gives up after about
// a second, sets MOE_ERR_TIMEOUT and lets the kernel run to its end without
// further work.
#pragma once

#include "common.cuh"
#include "router.cuh"
#include "tiledot.cuh"

namespace moeq {

constexpr int kStackMaxLayers = 64;
constexpr int kCWarps = 16;                      // compute warps
constexpr int kCThreads = kCWarps * 32;
constexpr int kStackThreads = kCThreads + 32;    // + producer warp
// The compute warp that publishes a phase's results (the release-add of a
// grid exchange waits until the CTA's writes are acknowledged, so it falls to
// the last warp, which takes a piece of the next phase last or not at all).
constexpr int kSigWarp = kCWarps - 1;
constexpr int kMaxSlots = 16;
constexpr int kMaxRouterRowsPerCta = 8;
constexpr int kRouterPieces = 4;                 // a router row is dotted in quarters
// (a CTA holds 3 or 4 routed gate/up tiles: 4 pieces each fill the 16 warps;
// 8 pieces, a shorter tail after the last tile lands, measured no faster)
#ifndef MOEQ_STACK_ROUTED_PIECES
#define MOEQ_STACK_ROUTED_PIECES 4
#endif
constexpr int kGuPieces = MOEQ_STACK_ROUTED_PIECES;  // pieces of a routed gate/up tile (half per ring item)
// pieces of a shared-expert gate/up tile: a CTA holds at most one or two of
// them, so four pieces would leave most warps idle before the top-K
#ifndef MOEQ_STACK_SHARED_PIECES
#define MOEQ_STACK_SHARED_PIECES 8
#endif
constexpr int kGuPiecesShared = MOEQ_STACK_SHARED_PIECES;
constexpr int kDnPieces = 4;                     // pieces of a (down tile, slot) job
constexpr int kMaxDnTiles = 4;                   // down tiles per CTA
constexpr int kItemPieces = kDnPieces * kMaxDnTiles;  // pieces of the largest item (a down item)
static_assert(kGuPiecesShared % 2 == 0 && kGuPiecesShared / 2 <= kItemPieces && kGuPieces % 2 == 0 &&
                  kGuPieces / 2 <= kItemPieces,
              "a ring item holds half of a tile's pieces");
constexpr int kMaxItems = 32;
constexpr int kMaxPieces = kMaxItems * kItemPieces;
constexpr int kMaxTiles = 16;                    // gate/up tiles per CTA per layer
constexpr int kStackMaxCtas = 1024;              // CTAs of the grid at most (partial sums in the workspace)
constexpr int kStackMaxE = 1024;                 // experts at most (two logits per compute thread)
// counters in the workspace: logits, shared h, routed h, r
enum { kSyncLogits = 0, kSyncSharedH = 1, kSyncRoutedH = 2, kSyncResid = 3, kNumSync };
static_assert(kNumSync <= 8, "arrival counters of the control block");

enum { kItemRouter = 0, kItemGateUp = 1, kItemDown = 2 };

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
  float* r;                 // [H] residual stream
  unsigned* sync;           // [4] arrival counters (kSync*)
  float* ss_part;           // [G] each CTA's sum of squares of its rows of r
  unsigned long long* trace;  // per-phase timestamps (builds with MOEQ_STACK_TRACE only), or null
  // shared-memory plan (byte offsets into the dynamic buffer)
  int sm_xs, sm_xplanes, sm_xgs;
  int sm_hplanes, hplanes_stride, sm_hgs, hgs_stride;
  int sm_gpart, sm_dpart, sm_ring, slot_bytes, nslot;
};

// Optional phase timeline (compiled in with -DMOEQ_STACK_TRACE only): one
// thread per CTA stamps %globaltimer at phase ends into
// trace[(layer * kTracePhases + phase) * G + cta]. Off in the library build.
// 14, 15: first/last routed gate/up item landed; 16: longest such piece (ns);
// 17, 18: routed h counter seen / its loads back; 19, 20: x staging loads
// back / image written; 21: the routed h arrival made; 22, 23: the copy
// warp done issuing layer l's routed items / the next layer's items;
// 24, 25: first routed down piece started / last one done; 26: longest such
// piece (ns)
constexpr int kTracePhases = 27;
#ifdef MOEQ_STACK_TRACE
#define STACK_MARK(cond, l, ph)                                                                    \
  do {                                                                                             \
    if ((cond) && p.trace) {                                                                       \
      unsigned long long t_;                                                                       \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                       \
      p.trace[((size_t)(l) * kTracePhases + (ph)) * gridDim.x + blockIdx.x] = t_;                  \
    }                                                                                              \
  } while (0)
#else
#define STACK_MARK(cond, l, ph) \
  do {                          \
  } while (0)
#endif

// CTA c's share [lo, hi) of n items split evenly over G CTAs.
// (n * c stays below 2^32: n is at most E, H/16 or K*I/8 of a plan that fits
// the kernel's tables, c at most kStackMaxCtas; 32-bit division keeps the
// plan's code short)
__host__ __device__ inline int share_lo(int c, int G, int n) { return (int)((unsigned)n * (unsigned)c / (unsigned)G); }
// Groups [lo, hi) of quarter q of a tile with ng groups.
__host__ __device__ inline int quarter_lo(int q, int ng) { return q * ng / 4; }

// The static item plan of one CTA (identical for every layer).
struct ItemPlan {
  int n_items, n_router_items, n_sgu_items, n_pre_items, n_rgu_items;  // item ranges, in ring order:
  // [0, n_router_items) router, [.., n_sgu_items) shared gate/up, [.., n_pre_items)
  // shared down (all three issued during the previous layer), [.., n_rgu_items)
  // routed gate/up, [.., n_items) routed down
  int n_pieces, n_router_pieces, n_pre_pieces;
  int kind[kMaxItems];
  int k[kMaxItems];                        // slot (K: shared)
  int tile[kMaxItems];                     // gate/up tile within its slot; router: first row (CTA-local)
  int tl[kMaxItems];                       // CTA-local gate/up tile index
  int half[kMaxItems];                     // which half of the tile's groups
  int npieces[kMaxItems];
  int piece0[kMaxItems];
  int nst;                                 // shared gate/up tiles (CTA-local tiles 0..nst-1)
  int r0, nr;                              // router rows [r0, r0+nr)
  int d0, nd;                              // down tiles [d0, d0+nd)
  int ntiles;
};

__device__ void make_plan(const StackParams& p, ItemPlan& P) {
  const int c = blockIdx.x, G = gridDim.x;
  int n = 0, pc = 0, tl = 0;
  P.r0 = share_lo(c, G, p.E);
  P.nr = share_lo(c + 1, G, p.E) - P.r0;
#pragma unroll 1
  for (int r = 0; r < P.nr; r += 2) {
    P.kind[n] = kItemRouter;
    P.k[n] = 0;
    P.tile[n] = r;
    P.tl[n] = 0;
    P.half[n] = 0;
    P.npieces[n] = kRouterPieces * min(2, P.nr - r);
    P.piece0[n] = pc;
    pc += P.npieces[n];
    ++n;
  }
  P.n_router_pieces = pc;
  P.n_router_items = n;
  auto add_tile = [&](int k, int T) {
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      P.kind[n] = kItemGateUp;
      P.k[n] = k;
      P.tile[n] = T;
      P.tl[n] = tl;
      P.half[n] = h;
      P.npieces[n] = k == p.K ? kGuPiecesShared / 2 : kGuPieces / 2;
      P.piece0[n] = pc;
      pc += P.npieces[n];
      ++n;
    }
    ++tl;
  };
  P.d0 = share_lo(c, G, p.H / kTileRows);
  P.nd = share_lo(c + 1, G, p.H / kTileRows) - P.d0;
  auto add_down = [&](int k) {
    P.kind[n] = kItemDown;
    P.k[n] = k;
    P.tile[n] = 0;
    P.tl[n] = 0;
    P.half[n] = 0;
    P.npieces[n] = kDnPieces * P.nd;
    P.piece0[n] = pc;
    pc += P.npieces[n];
    ++n;
  };
  const int tps = p.I / 8;  // gate/up tiles per slot
#pragma unroll 1
  for (int T = share_lo(c, G, tps); T < share_lo(c + 1, G, tps); ++T) add_tile(p.K, T);
  P.nst = tl;
  P.n_sgu_items = n;
  if (P.nd > 0) add_down(p.K);
  P.n_pre_items = n;
  P.n_pre_pieces = pc;
#pragma unroll 1
  for (int u = share_lo(c, G, p.K * tps); u < share_lo(c + 1, G, p.K * tps); ++u) add_tile(u / tps, u % tps);
  P.n_rgu_items = n;
  if (P.nd > 0)
#pragma unroll 1
    for (int k = 0; k < p.K; ++k) add_down(k);
  P.n_items = n;
  P.n_pieces = pc;
  P.ntiles = tl;
}

// ---- producer pieces ---------------------------------------------------------

struct Ring {
  uint64_t* full;
  uint64_t* empty;
  int* last;     // per slot: ring sequence number of the last fill issued (-1: none)
  unsigned char* base;
  int slot_bytes, nslot;
};

// Source and size of ring item `it` of layer l (0 bytes: an empty item, for
// a slot whose expert index was invalid).
__device__ __forceinline__ uint32_t item_source(const StackParams& p, const ItemPlan& P, int l, int it,
                                                const int* s_idx, const void** src) {
  if (P.kind[it] == kItemRouter) {
    *src = p.L[l].router_w + (size_t)(P.r0 + P.tile[it]) * p.H;
    return (uint32_t)(P.npieces[it] / kRouterPieces) * (uint32_t)p.H * 2;
  }
  const int k = P.k[it];
  const RecGeom& g = k == p.K ? p.geo_s : p.geo_r;
  const uint8_t* rec;
  if (k == p.K) {
    rec = p.L[l].shared;
  } else {
    const int e = s_idx[k];
    if (e < 0) return 0u;
    rec = p.L[l].experts + (size_t)e * p.rec_r;
  }
  if (P.kind[it] == kItemDown) {
    *src = rec + g.down_off + (size_t)P.d0 * g.D;
    return (uint32_t)P.nd * g.D;
  }
  const int ga = quarter_lo(2 * P.half[it], (int)g.ng_h), gb = quarter_lo(2 * P.half[it] + 2, (int)g.ng_h);
  *src = rec + (size_t)P.tile[it] * g.U + (size_t)ga * g.blk;
  return (uint32_t)(gb - ga) * g.blk;
}

// Issue ring items [it0, it1) of layer l, item it taking ring sequence number
// seq0 + (it - it0). A thread's bulk copies go out one after another, so the
// lanes issue in parallel: each round takes the run of next items whose slots
// are already free (lane j -> item next + j); if none is, lane 0 waits for
// the first. Returns false if a wait gave up.
__device__ bool issue_items(const StackParams& p, const ItemPlan& P, Ring& R, int l, int it0, int it1, uint32_t seq0,
                            const int* s_idx, const volatile int* abort, long long budget) {
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
      if (lane == 0) ok = mbar_wait(&R.empty[slot], (fill - 1) & 1, abort, budget);
      if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) return false;
      nr = 1;
    }
    if (lane < nr) {
      const void* src = nullptr;
      const uint32_t bytes = item_source(p, P, l, next + lane, s_idx, &src);
      *reinterpret_cast<volatile int*>(&R.last[slot]) = (int)seq;
      mbar_arrive_expect_tx(&R.full[slot], bytes);
      if (bytes) bulk_g2s(R.base + (size_t)slot * R.slot_bytes, src, bytes, &R.full[slot]);
    }
    __syncwarp();
    next += nr;
  }
  return true;
}

// ---- softmax and top-K -------------------------------------------------------

// Bounded wait until the shared-memory flag reaches target.
__device__ __forceinline__ bool flag_wait(const volatile int* f, int target, const volatile int* abort,
                                          long long budget) {
  if (*f >= target) return true;
  const long long t0 = clock64();
  while (*f < target) {
    if (*abort || clock64() - t0 > budget) return false;
    __nanosleep(32);
  }
  return true;
}

// The sum of the G CTAs' published partial sums of squares by one warp, in
// one fixed order (lane j adds entries j, j+32, ... then a butterfly over the
// lanes), so every CTA gets the same value. The loads are all issued before
// the first add (one L2 round trip for G <= 256).
__device__ __forceinline__ float sum_partials(const float* part, int G) {
  const int lane = threadIdx.x & 31;
  float v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = lane + 32 * j < G ? __ldcg(part + lane + 32 * j) : 0.f;
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += v[j];
  for (int c = lane + 256; c < G; c += 32) s += __ldcg(part + c);
  return warp_sum(s);
}

// ---- compute pieces ------------------------------------------------------------

// Bounded wait until the producer has issued ring sequence number seq into
// `slot` (it records that before arming the slot's full barrier). The copy
// still has to land after that, so the pause between looks can be long.
__device__ __forceinline__ bool slot_issued(const int* last, int slot, int seq, const volatile int* abort,
                                            long long budget) {
  const volatile int* v = last;
  if (v[slot] == seq) return true;
  const long long t0 = clock64();
  while (v[slot] != seq) {
    if (*abort || clock64() - t0 > budget) return false;
    __nanosleep(200);
  }
  return true;
}

__device__ __forceinline__ QImg stack_himg(unsigned char* sm, const StackParams& p, int k) {
  return QImg{reinterpret_cast<uint2*>(sm + p.sm_hplanes + (size_t)k * p.hplanes_stride),
              reinterpret_cast<float2*>(sm + p.sm_hgs + (size_t)k * p.hgs_stride)};
}

// One kernel per format (BR bits routed, BS bits shared, KS k-steps per
// group): the host picks the instance for the layers' widths and group.
template <int BR, int BS, int KS>
__global__ void __launch_bounds__(kStackThreads, 1) k_decode_layers(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t full_bar[kMaxSlots], empty_bar[kMaxSlots];
  __shared__ int s_last[kMaxSlots];
  __shared__ int s_idx[MOEQ_MAX_K];
  __shared__ float s_w[MOEQ_MAX_K];
  __shared__ float s_rpart[kMaxRouterRowsPerCta][kRouterPieces];
  __shared__ int s_gcnt[kMaxTiles];
  __shared__ float s_red[2][kCWarps];
  __shared__ unsigned char s_piece_item[kMaxPieces];
  __shared__ ItemPlan P;
  __shared__ SelScratch<kCWarps> s_topk;
  __shared__ volatile int s_abort;
  __shared__ volatile int s_topk_ready;
  __shared__ volatile int s_logits_ready;  // layer + 1 once s_logits holds that layer's logits
  __shared__ volatile int s_rh_arrived;    // layer + 1 once this CTA's routed h arrival is made
  __shared__ float s_inv_norm;             // 1 / RMS of r_l (x staging)
#ifdef MOEQ_STACK_TRACE
  __shared__ unsigned long long s_tr[6];
  if (threadIdx.x == 0) {
    s_tr[0] = s_tr[3] = ~0ull;
    s_tr[1] = s_tr[2] = s_tr[4] = s_tr[5] = 0ull;
  }
#endif
  __shared__ __align__(16) float s_logits[kStackMaxE];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x;
  const long long budget = wait_budget(p.ctrl);
  // testing hook: this CTA skips its first logits arrival, so every CTA's
  // logits wait runs out of budget (a fault made on the host, never on the GPU)
  const bool withhold = *reinterpret_cast<const volatile int*>(&p.ctrl->withhold_cta) == (int)blockIdx.x + 1;

  if (tid == 0) {
    make_plan(p, P);
#pragma unroll 1
    for (int it = 0; it < P.n_items; ++it)
#pragma unroll 1
      for (int q = 0; q < P.npieces[it]; ++q) s_piece_item[P.piece0[it] + q] = (unsigned char)it;
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kItemPieces);
      s_last[i] = -1;
    }
    for (int t = 0; t < kMaxTiles; ++t) s_gcnt[t] = 0;
    s_abort = 0;
    s_topk_ready = 0;
    s_logits_ready = 0;
    s_rh_arrived = 0;
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
    if (!issue_items(p, P, R, 0, 0, P.n_pre_items, 0u, s_idx, &s_abort, budget) && lane == 0) fail();
    for (int l = 0; l < p.n_layers; ++l) {
      // relay: once every CTA has published layer l's logits, copy them into
      // shared memory for the compute warps' top-K (the poll and the L2 read
      // overlap the compute warps' shared-expert work)
      if (lane == 0 && !s_abort && !counter_wait(p.sync + kSyncLogits, (unsigned)(l + 1) * (unsigned)G, &s_abort, budget) &&
          !s_abort)
        fail();
      __syncwarp();
      for (int e = lane; e < p.E; e += 32) s_logits[e] = __ldcg(p.logits + e);
      __syncwarp();
      __threadfence_block();
      if (lane == 0) s_logits_ready = l + 1;
      // routing: the compute warps publish layer l's picks in s_idx/s_w
      if (lane == 0 && !s_abort && !flag_wait(&s_topk_ready, l + 1, &s_abort, budget) && !s_abort) fail();
      __syncwarp();
      __threadfence_block();
      STACK_MARK(lane == 0, l, 13);
      // routed gate/up items (they gate the h exchange), the routed down
      // items (needed only after it), then the next layer's router, shared
      // gate/up and shared down items. What follows the gate/up items waits
      // for this CTA's routed h arrival: a gpu-scope release waits for the
      // CTA's bulk copies in flight, so copies issued before it would hold
      // up the arrival that every CTA waits for.
      const uint32_t seq_l = (uint32_t)(l * n_items);
#if MOEQ_STACK_HOLD_DOWN
      bool ok = !s_abort && issue_items(p, P, R, l, P.n_pre_items, P.n_rgu_items, seq_l + P.n_pre_items, s_idx,
                                        &s_abort, budget);
      if (ok && lane == 0 && !flag_wait(&s_rh_arrived, l + 1, &s_abort, budget) && !s_abort) fail();
      __syncwarp();
      ok = ok && !s_abort &&
           issue_items(p, P, R, l, P.n_rgu_items, n_items, seq_l + P.n_rgu_items, s_idx, &s_abort, budget);
      STACK_MARK(lane == 0, l, 22);
#else
      bool ok = !s_abort && issue_items(p, P, R, l, P.n_pre_items, n_items, seq_l + P.n_pre_items, s_idx, &s_abort, budget);
      STACK_MARK(lane == 0, l, 22);
      if (ok && l + 1 < p.n_layers && lane == 0 && !flag_wait(&s_rh_arrived, l + 1, &s_abort, budget) && !s_abort) fail();
      __syncwarp();
#endif
      if (ok && l + 1 < p.n_layers)
        ok = issue_items(p, P, R, l + 1, 0, P.n_pre_items, (uint32_t)((l + 1) * n_items), s_idx, &s_abort, budget);
      STACK_MARK(lane == 0, l, 23);
      if (!ok && lane == 0 && !s_abort) fail();
      __syncwarp();
    }
    // drain: every copy issued must have landed before the CTA exits
    if (lane < p.nslot) {
      const int j = s_last[lane];
      if (j >= 0) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&full_bar[lane], (j / p.nslot) & 1) && clock64() - t0 < budget) {
        }
      }
    }
    __syncwarp();
  } else {
    // ===================== compute warps =====================
    const int H = p.H, I = p.I, K = p.K;
    uint16_t* xs = reinterpret_cast<uint16_t*>(sm + p.sm_xs);
    const QImg X{reinterpret_cast<uint2*>(sm + p.sm_xplanes), reinterpret_cast<float2*>(sm + p.sm_xgs)};
    float* gpart = reinterpret_cast<float*>(sm + p.sm_gpart);  // [tile][4][16]
    float* dpart = reinterpret_cast<float*>(sm + p.sm_dpart);  // [tile][K+1][4][16]
    const unsigned char* ring = sm + p.sm_ring;
    // the thread's output row (combine), carried across layers
    const int my_row = tid < P.nd * kTileRows ? P.d0 * kTileRows + tid : -1;
    float my_r = 0.f;
    if (my_row >= 0) my_r = p.resid_in ? p.resid_in[my_row] : bf16_bits_to_f32(p.x_in[my_row]);

    // One piece of the ring: a router quarter-row or a gate/up quarter-tile.
    // Compute warps may run several fills ahead of a slot, so a piece first
    // waits until the producer has issued its fill: only then does the full
    // barrier's parity name that fill and not an older one.
    auto do_piece = [&](int l, int pc) {
      const int it = s_piece_item[pc];
      const int pos = pc - P.piece0[it];
      const uint32_t seq = (uint32_t)(l * n_items + it);
      const int slot = seq % p.nslot;
      bool ok = slot_issued(s_last, slot, (int)seq, &s_abort, budget);
      ok = ok && mbar_wait(&full_bar[slot], (seq / p.nslot) & 1, &s_abort, budget);
      if (!ok && lane == 0 && !s_abort) fail();
#ifdef MOEQ_STACK_TRACE
      unsigned long long t_landed = 0;
      const bool traced = it >= P.n_pre_items && it < P.n_rgu_items;
      if (traced && lane == 0) {
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_landed));
        atomicMin(&s_tr[0], t_landed);
        atomicMax(&s_tr[1], t_landed);
      }
#endif
      const unsigned char* sl = ring + (size_t)slot * p.slot_bytes;
      if (P.kind[it] == kItemRouter) {
        const int row = pos / kRouterPieces, qr = pos % kRouterPieces;
        const int nv = H / (8 * kRouterPieces);  // 16-byte words in a quarter row
        const uint4* wv = reinterpret_cast<const uint4*>(sl + (size_t)row * H * 2) + qr * nv;
        const uint4* xv = reinterpret_cast<const uint4*>(xs) + qr * nv;
        float acc = 0.f;
        if (ok)
          for (int v = lane; v < nv; v += 32) acc = dot8_bf16(wv[v], xv[v], acc);
        acc = warp_sum(acc);
        if (lane == 0) s_rpart[P.tile[it] + row][qr] = acc;
      } else if (P.kind[it] == kItemDown) {
#ifdef MOEQ_STACK_TRACE
        unsigned long long t_dn0 = 0;
        if (P.k[it] < K && lane == 0) asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_dn0));
#endif
        const int k = P.k[it], q = pos % kDnPieces, j = pos / kDnPieces;
        const bool routed = k < K;
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int g0 = quarter_lo(q, (int)g.ng_i), g1 = quarter_lo(q + 1, (int)g.ng_i);
        float acc0 = 0.f, acc1 = 0.f;
        if (ok && (!routed || s_idx[k] >= 0)) {
          const unsigned char* blk = sl + (size_t)j * g.D + (size_t)g0 * g.blk;
          const QImg Hk = stack_himg(sm, p, k);
          with_fixed_fmt<BR, BS, KS>(
              routed, [&]<int BITS, int KS_>() { tile_dot<BITS, KS_>(blk, g1 - g0, g0, Hk, acc0, acc1); });
        }
        if ((lane & 3) == 0) {
          float* dp = dpart + (((size_t)j * (K + 1) + k) * kDnPieces + q) * kTileRows;
          dp[lane >> 2] = acc0;
          dp[(lane >> 2) + 8] = acc1;
        }
#ifdef MOEQ_STACK_TRACE
        if (routed && lane == 0) {
          unsigned long long t_dn1;
          asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_dn1));
          atomicMin(&s_tr[3], t_dn0);
          atomicMax(&s_tr[4], t_dn1);
          atomicMax(&s_tr[5], t_dn1 - t_dn0);
        }
#endif
      } else {
        const int k = P.k[it], tl = P.tl[it], npi = P.npieces[it], npt = 2 * npi, q = npi * P.half[it] + pos;
        const bool routed = k < K;
        const bool valid = ok && (!routed || s_idx[k] >= 0);
        const RecGeom& g = routed ? p.geo_r : p.geo_s;
        const int ng = (int)g.ng_h;
        const int ga = quarter_lo(2 * P.half[it], ng);
        const int g0 = q * ng / npt, g1 = (q + 1) * ng / npt;
        // the tile's partial sums: shared tiles (first) hold kGuPiecesShared pieces, routed ones kGuPieces
        float* g4 = gpart + (tl < P.nst ? (size_t)tl * kGuPiecesShared
                                        : (size_t)P.nst * kGuPiecesShared + (size_t)(tl - P.nst) * kGuPieces) *
                                kTileRows;
        float acc0 = 0.f, acc1 = 0.f;
        if (valid) {
          const unsigned char* blk = sl + (size_t)(g0 - ga) * g.blk;
          with_fixed_fmt<BR, BS, KS>(
              routed, [&]<int BITS, int KS_>() { tile_dot<BITS, KS_>(blk, g1 - g0, g0, X, acc0, acc1); });
        }
        float* gp = g4 + (size_t)q * kTileRows;
        if ((lane & 3) == 0) {
          gp[lane >> 2] = acc0;
          gp[(lane >> 2) + 8] = acc1;
          __threadfence_block();
        }
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(&s_gcnt[tl], 1);
        prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
        if (prev == npt - 1) {  // the tile's last piece: finish its 8 units
          __threadfence_block();
          if (lane < 8) {
            float gate = 0.f, up = 0.f;
            for (int qq = 0; qq < npt; ++qq) {
              gate += g4[qq * kTileRows + lane];
              up += g4[qq * kTileRows + 8 + lane];
            }
            const float hv = (!routed || s_idx[k] >= 0) ? silu_f(gate) * up : 0.f;
            __stcg(p.h + (size_t)k * I + 8 * P.tile[it] + lane, hv);
          }
          if (lane == 0) s_gcnt[tl] = 0;
        }
      }
      __syncwarp();
#ifdef MOEQ_STACK_TRACE
      if (traced && lane == 0) {
        unsigned long long t_done;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_done));
        atomicMax(&s_tr[2], t_done - t_landed);
      }
#endif
      if (lane == 0) {
        const uint32_t cnt = (pos == 0) ? (uint32_t)(kItemPieces - P.npieces[it] + 1) : 1u;
        mbar_arrive_cnt(&empty_bar[slot], cnt);
      }
    };

    // The pieces of ring items [it0, it1), spread over the compute warps.
    auto run_items = [&](int l, int it0, int it1) {
      if (it1 <= it0) return;
      const int pc1 = P.piece0[it1 - 1] + P.npieces[it1 - 1];
      for (int pc = P.piece0[it0] + warp; pc < pc1; pc += kCWarps) do_piece(l, pc);
    };

    // Stage the h_k images of slots [k0, k1) once every CTA has counted its
    // part of them out (counter `c` at `target`). Each lane stages its own
    // segment into its own slot's image; a group's lanes are adjacent and
    // share a slot (I is a multiple of G).
    auto stage_h = [&](int l, int k0, int k1, int c, unsigned target) {
      if (tid == 0 && !counter_wait(p.sync + c, target, &s_abort, budget) && !s_abort) fail();
      STACK_MARK(tid == 0 && k0 == 0, l, 17);
      named_sync(1, kCThreads);
      const int spk = I / 16;  // segments per slot
      for (int s0 = tid - lane; s0 < (k1 - k0) * spk; s0 += kCThreads) {
        const int s = s0 + lane;
        const bool active = s < (k1 - k0) * spk;
        const int k = active ? k0 + s / spk : k0, sk = active ? s % spk : 0;
        float v[16];
        if (active) {
          load_f32_16_cg(p.h + (size_t)k * I + (size_t)sk * 16, v);
          STACK_MARK(tid == 0 && k0 == 0 && s0 == 0 && v[0] == v[0], l, 18);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
        }
        qstage_seg(v, sk, p.G, stack_himg(sm, p, k), active);
      }
    };

    const unsigned G1 = (unsigned)G;
    for (int l = 0; l < p.n_layers; ++l) {
      STACK_MARK(tid == 0, l, 0);
      // ---- stage x_l ----
      {
        const uint16_t* gw = p.L[l].gate_w;
        const int nseg = H / 16;
        float v[16];
        const bool active = tid < nseg;
        if (l > 0) {
          if (tid == 0 && !counter_wait(p.sync + kSyncResid, (unsigned)l * G1, &s_abort, budget) && !s_abort) fail();
          STACK_MARK(tid == 0, l, 1);
          named_sync(1, kCThreads);
          // the RMS norm's sum of squares from the CTAs' published partial
          // sums, in one fixed order (every CTA gets the same value), read by
          // one warp in the same round trip as r (one reader per CTA of those
          // few lines instead of sixteen)
          if (active) load_f32_16_cg(p.r + (size_t)tid * 16, v);
          if (warp == 0) {
            const float t = sum_partials(p.ss_part, G);
            if (lane == 0) s_inv_norm = rsqrtf(t / (float)H + p.eps);
          }
          named_sync(1, kCThreads);
          const float inv_norm = s_inv_norm;
          STACK_MARK(tid == 0 && v[0] == v[0], l, 19);
          if (active) {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = bf16_bits_to_f32(f32_to_bf16_bits(v[j] * inv_norm));
          }
        } else if (active) {
          load_bf16_16(p.x_in + (size_t)tid * 16, v);
        }
        float gdot = 0.f;
        if (active) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              w[i] = (__float_as_uint(v[8 * q + 2 * i]) >> 16) | (__float_as_uint(v[8 * q + 2 * i + 1]) & 0xFFFF0000u);
            reinterpret_cast<uint4*>(xs + (size_t)tid * 16)[q] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (gw) {
            float gv[16];
            load_bf16_16(gw + (size_t)tid * 16, gv);
#pragma unroll
            for (int j = 0; j < 16; ++j) gdot += gv[j] * v[j];
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
        }
        if (warp * 32 < nseg) qstage_seg(v, tid, p.G, X, active);
        STACK_MARK(tid == 0, l, 20);
        gdot = warp_sum(gdot);
        if (lane == 0) s_red[1][warp] = gdot;
        named_sync(1, kCThreads);
      }
      STACK_MARK(tid == 0, l, 2);
      float gamma = 1.f;
      if (p.L[l].gate_w) {
        float d = 0.f;
        for (int w = 0; w < kCWarps; ++w) d += s_red[1][w];
        gamma = 1.f / (1.f + expf(-d));
      }

      // ---- router pieces, then the shared expert's gate/up pieces ----
      run_items(l, 0, P.n_router_items);
      named_sync(1, kCThreads);
      if (warp == kSigWarp) {
        if (lane < P.nr) {
          float lg = 0.f;
#pragma unroll
          for (int qr = 0; qr < kRouterPieces; ++qr) lg += s_rpart[lane][qr];
          __stcg(p.logits + P.r0 + lane, lg);
        }
        __syncwarp();
        if (lane == 0 && !(withhold && l == 0)) arrive_release_gpu(p.sync + kSyncLogits);
      }
      STACK_MARK(tid == 0, l, 3);
      run_items(l, P.n_router_items, P.n_sgu_items);
      named_sync(1, kCThreads);
      if (tid == kSigWarp * 32) arrive_release_gpu(p.sync + kSyncSharedH);
      STACK_MARK(tid == 0, l, 4);

      // ---- softmax / top-K over every CTA's logits (the producer waits for it) ----
      if (lane == 0 && !flag_wait(&s_logits_ready, l + 1, &s_abort, budget) && !s_abort) fail();
      __syncwarp();
      STACK_MARK(tid == 0, l, 5);
      {  // (all compute warps; warp 0 ends with the picks and weights)
        const int32_t* forced = p.forced ? p.forced + (size_t)l * K : nullptr;
        block_select<kCWarps, kStackMaxE / kCThreads>(s_logits, p.E, K, p.renorm, forced, s_topk,
                                                       [] { named_sync(1, kCThreads); }, s_idx, s_w, p.ctrl);
        if (warp == 0) {
          __syncwarp();
          if (blockIdx.x == 0 && lane < K) {
            if (p.idx_out) p.idx_out[(size_t)l * K + lane] = forced ? forced[lane] : s_idx[lane];
            if (p.w_out) p.w_out[(size_t)l * K + lane] = s_w[lane];
          }
          __syncwarp();
          __threadfence_block();
          if (lane == 0) s_topk_ready = l + 1;
        }
      }
      STACK_MARK(tid == 0, l, 6);

      // ---- the shared expert's down tiles, once every CTA's shared h is out ----
      stage_h(l, K, K + 1, kSyncSharedH, (unsigned)(l + 1) * G1);
      named_sync(1, kCThreads);
      STACK_MARK(tid == 0, l, 7);
      run_items(l, P.n_sgu_items, P.n_pre_items);
      STACK_MARK(tid == 0, l, 8);

      // ---- routed gate/up pieces ----
      run_items(l, P.n_pre_items, P.n_rgu_items);
      named_sync(1, kCThreads);
      if (tid == kSigWarp * 32) {
        arrive_release_gpu(p.sync + kSyncRoutedH);
        s_rh_arrived = l + 1;
      }
      STACK_MARK(tid == kSigWarp * 32, l, 21);
      STACK_MARK(tid == 0, l, 9);
#ifdef MOEQ_STACK_TRACE
      if (tid == 0 && p.trace) {
        const size_t at = (size_t)l * kTracePhases * gridDim.x + blockIdx.x;
        p.trace[at + (size_t)14 * gridDim.x] = s_tr[0];
        p.trace[at + (size_t)15 * gridDim.x] = s_tr[1];
        p.trace[at + (size_t)16 * gridDim.x] = s_tr[2];
        s_tr[0] = ~0ull;
        s_tr[1] = 0ull;
        s_tr[2] = 0ull;
      }
#endif

      // ---- routed down tiles ----
      stage_h(l, 0, K, kSyncRoutedH, (unsigned)(l + 1) * G1);
      named_sync(1, kCThreads);
      STACK_MARK(tid == 0, l, 10);
      run_items(l, P.n_rgu_items, n_items);
      named_sync(1, kCThreads);
      STACK_MARK(tid == 0, l, 11);
#ifdef MOEQ_STACK_TRACE
      if (tid == 0 && p.trace) {
        const size_t at = (size_t)l * kTracePhases * gridDim.x + blockIdx.x;
        p.trace[at + (size_t)24 * gridDim.x] = s_tr[3];
        p.trace[at + (size_t)25 * gridDim.x] = s_tr[4];
        p.trace[at + (size_t)26 * gridDim.x] = s_tr[5];
        s_tr[3] = ~0ull;
        s_tr[4] = 0ull;
        s_tr[5] = 0ull;
      }
#endif

      // ---- combine: r_{l+1} = r_l + sum_k w_k y_k + gamma y_shared ----
      if (my_row >= 0) {
        const int j = tid / kTileRows, rho = tid % kTileRows;
        float y = 0.f;
        for (int k = 0; k <= K; ++k) {
          const float wk = k < K ? (s_idx[k] >= 0 ? s_w[k] : 0.f) : gamma;
          const float* dp = dpart + (((size_t)j * (K + 1) + k) * kDnPieces) * kTileRows + rho;
          float yk = 0.f;
#pragma unroll
          for (int q = 0; q < kDnPieces; ++q) yk += dp[q * kTileRows];
          y += wk * yk;
        }
        my_r += y;
        if (l + 1 < p.n_layers || p.xnorm_out) __stcg(p.r + my_row, my_r);
        if (l + 1 == p.n_layers) p.resid_out[my_row] = my_r;
      }
      {  // this CTA's partial sum of squares of r_{l+1}, published with its rows
        const float sq = warp_sum(my_row >= 0 ? my_r * my_r : 0.f);
        if (lane == 0) s_red[0][warp] = sq;
      }
      named_sync(1, kCThreads);
      if (tid == kSigWarp * 32) {
        float t = 0.f;
        for (int w = 0; w < kCWarps; ++w) t += s_red[0][w];
        __stcg(p.ss_part + blockIdx.x, t);
        arrive_release_gpu(p.sync + kSyncResid);
      }
      STACK_MARK(tid == 0, l, 12);
    }

    // ---- optional RMSNorm'd bf16 output of the last layer ----
    if (p.xnorm_out) {
      const int nseg = H / 16;
      float ss = 0.f;
      if (tid == 0 && !counter_wait(p.sync + kSyncResid, (unsigned)p.n_layers * G1, &s_abort, budget) && !s_abort) fail();
      named_sync(1, kCThreads);
      (void)nseg;
      (void)ss;
      if (warp == 0) {
        const float t = sum_partials(p.ss_part, G);
        if (lane == 0) s_inv_norm = rsqrtf(t / (float)H + p.eps);
      }
      named_sync(1, kCThreads);
      const float inv = s_inv_norm;
      if (my_row >= 0) p.xnorm_out[my_row] = f32_to_bf16_bits(my_r * inv);
    }
  }

  // ---- leave: the last CTA out resets the counters ----
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned t = atomicAdd(&p.ctrl->exit_count, 1u);
    if (t == (unsigned)G - 1) {
      for (int c = 0; c < kNumSync; ++c) atomicExch(p.sync + c, 0u);
      __threadfence();
      atomicExch(&p.ctrl->exit_count, 0u);
    }
  }
}

}  // namespace moeq
