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
//   router         CTA c owns router rows c, c+G, ...; writes its logits
//   sync 1         all logits written
//   top-K          the producer warp of every CTA selects the K experts
//   gate/up        shared-expert units (slot K, row i) and routed units
//                  (slot k, row i), strided over the CTAs; h to global
//   sync 2         all of h written
//   down+combine   CTA c owns output row blocks c, c+G, ... (4 rows): for
//                  every slot the row dot with h_k, weighted by the routing
//                  weight (shared: gamma), plus the residual
//   sync 3         r_{l+1} and its sum of squares complete
//
// Warp roles: warps 0..7 compute, warp 8 moves data. The producer streams
// every weight byte of the CTA's share into shared memory with bulk async
// copies (cp.async.bulk, completion on mbarriers): router half-rows and
// gate/up units through a ring of slots, down-projection row blocks into a
// region that is filled as soon as the experts are known, so down weights
// arrive while gate/up still computes. Router rows and shared-expert units of
// layer l+1 enter the ring while layer l finishes. Grid-wide syncs are
// monotonic arrival counters in the workspace; every wait (counter or
// mbarrier) gives up after about a second, sets MOE_ERR_TIMEOUT and lets the
// kernel run to its end without further work.
#pragma once

#include "common.cuh"
#include "ffn.cuh"
#include "router.cuh"

namespace moeq {

constexpr int kStackMaxLayers = 64;
constexpr int kCWarps = 8;                          // compute warps
constexpr int kCThreads = kCWarps * 32;
constexpr int kStackThreads = kCThreads + 32;       // + producer warp
constexpr int kDnBlk = 4;                           // rows per down block
constexpr int kMaxSlots = 32;
constexpr int kMaxRouterRowsPerCta = 8;

enum { kItemRouterHalf = 0, kItemGateUp = 1, kItemZero = 2 };

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
  uint32_t off_r[6], off_s[6];
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
  int sm_xs, sm_img4, sm_tab4, sm_img2, sm_tab2, sm_himg, sm_htab, himg_stride, htab_stride;
  int sm_ring, slot_bytes, nslot, sm_regc, dblk_bytes, nblk_max;
  int need4, need2;
};

__host__ __device__ inline int strided_count(int c, int G, int n) { return n > c ? (n - c - 1) / G + 1 : 0; }

// ---- producer pieces ---------------------------------------------------------

struct Ring {
  uint64_t* full;
  uint64_t* empty;
  int* kind;
  int* a;
  int* b;
  int* last;     // per slot: sequence number of the last fill actually issued (-1: none)
  unsigned char* base;
  int slot_bytes, nslot;
  uint32_t seq;  // items issued so far
};

// Issue one ring item (lane 0 copies, the whole warp waits for the slot).
__device__ __forceinline__ void ring_issue(Ring& R, int kind, int a, int b, const void* const* src,
                                           const uint32_t* bytes, int ncopy, const volatile int* abort) {
  const uint32_t slot = R.seq % R.nslot, n = R.seq / R.nslot;
  bool ok = true;
  if (n > 0) ok = mbar_wait(&R.empty[slot], (n - 1) & 1, abort);
  if ((threadIdx.x & 31) == 0) {
    if (ok) {
      R.kind[slot] = kind;
      R.a[slot] = a;
      R.b[slot] = b;
      R.last[slot] = (int)R.seq;
      uint32_t tot = 0;
      for (int i = 0; i < ncopy; ++i) tot += bytes[i];
      mbar_arrive_expect_tx(&R.full[slot], tot);
      unsigned char* dst = R.base + (size_t)slot * R.slot_bytes;
      for (int i = 0; i < ncopy; ++i) {
        bulk_g2s(dst, src[i], bytes[i], &R.full[slot]);
        dst += bytes[i];
      }
    }
  }
  __syncwarp();
  R.seq++;
}

// Router half-rows and shared-expert gate/up units of layer l (they do not
// depend on the routing).
__device__ void issue_pre(const StackParams& p, Ring& R, int l, int nr, int nsu, const volatile int* abort) {
  const int c = blockIdx.x, G = gridDim.x;
  const uint32_t half_bytes = (uint32_t)p.H;  // H/2 bf16
  for (int m = 0; m < nr; ++m) {
    const int e = c + G * m;
    for (int hh = 0; hh < 2; ++hh) {
      const void* src[1] = {p.L[l].router_w + (size_t)e * p.H + (size_t)hh * (p.H / 2)};
      const uint32_t by[1] = {half_bytes};
      ring_issue(R, kItemRouterHalf, m, hh, src, by, 1, abort);
    }
  }
  const uint32_t rowb = (uint32_t)(p.H * p.bits_s / 8), sbb = (uint32_t)(p.H / p.G * 4);
  for (int m = 0; m < nsu; ++m) {
    const int i = c + G * m;
    const uint8_t* rec = p.L[l].shared;
    const void* src[4] = {rec + p.off_s[0] + (size_t)i * rowb, rec + p.off_s[1] + (size_t)i * rowb,
                          rec + p.off_s[3] + (size_t)i * sbb, rec + p.off_s[4] + (size_t)i * sbb};
    const uint32_t by[4] = {rowb, rowb, sbb, sbb};
    ring_issue(R, kItemGateUp, p.K, i, src, by, 4, abort);
  }
}

// Routed gate/up units of layer l (needs the experts in s_idx).
__device__ void issue_routed(const StackParams& p, Ring& R, int l, int nru, const int* s_idx, const volatile int* abort) {
  const int c = blockIdx.x, G = gridDim.x;
  const uint32_t rowb = (uint32_t)(p.H * p.bits_r / 8), sbb = (uint32_t)(p.H / p.G * 4);
  for (int m = 0; m < nru; ++m) {
    const int u = c + G * m;
    const int k = u / p.I, i = u % p.I;
    const int e = s_idx[k];
    if (e < 0) {
      ring_issue(R, kItemZero, k, i, nullptr, nullptr, 0, abort);
      continue;
    }
    const uint8_t* rec = p.L[l].experts + (size_t)e * p.rec_r;
    const void* src[4] = {rec + p.off_r[0] + (size_t)i * rowb, rec + p.off_r[1] + (size_t)i * rowb,
                          rec + p.off_r[3] + (size_t)i * sbb, rec + p.off_r[4] + (size_t)i * sbb};
    const uint32_t by[4] = {rowb, rowb, sbb, sbb};
    ring_issue(R, kItemGateUp, k, i, src, by, 4, abort);
  }
}

// Down-projection row blocks of slot k (expert record `rec`, `bits`) into the
// down region; lane 0 only. Returns the bytes issued.
__device__ uint32_t issue_down_slot(const StackParams& p, unsigned char* regc, int k, const uint8_t* rec,
                                    const uint32_t* off, int bits, int nblk, uint64_t* bar, bool issue) {
  const int c = blockIdx.x, G = gridDim.x;
  const uint32_t rowb = (uint32_t)(p.I * bits / 8), sbb = (uint32_t)(p.I / p.G * 4);
  uint32_t tot = 0;
  for (int m = 0; m < nblk; ++m) {
    const int i0 = (c + G * m) * kDnBlk;
    unsigned char* dst = regc + ((size_t)k * p.nblk_max + m) * p.dblk_bytes;
    if (issue) {
      bulk_g2s(dst, rec + off[2] + (size_t)i0 * rowb, kDnBlk * rowb, bar);
      bulk_g2s(dst + kDnBlk * rowb, rec + off[5] + (size_t)i0 * sbb, kDnBlk * sbb, bar);
    }
    tot += kDnBlk * (rowb + sbb);
  }
  return tot;
}

// Top-K (or forced picks) of layer l by the producer warp, from the logits
// every CTA published. Writes s_idx (-1 for an invalid forced index) and s_w.
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
  for (int j = 0; j < MAXV; ++j)
    if (lane + 32 * j < p.E) z += expf(v[j] - mx);
  z = warp_sum(z);
  int picked[MOEQ_MAX_K];
  const int32_t* forced = p.forced ? p.forced + (size_t)l * p.K : nullptr;
  for (int k = 0; k < p.K; ++k) {
    if (forced) {
      const int e = forced[k];
      picked[k] = (e >= 0 && e < p.E) ? e : -1;
      if (picked[k] < 0 && lane == 0) set_error(p.ctrl, MOE_ERR_INDEX);
      continue;
    }
    float best = -INFINITY;
    int bi = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < MAXV; ++j) {
      const int e = lane + 32 * j;
      bool taken = false;
      for (int q = 0; q < k; ++q) taken |= (picked[q] == e);
      if (e < p.E && !taken && (v[j] > best || (v[j] == best && e < bi))) {
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
    if (bi < 0 || bi >= p.E) {  // no finite logit left (NaN input): no expert
      if (lane == 0) set_error(p.ctrl, MOE_ERR_INDEX);
      bi = -1;
    }
    picked[k] = bi;
  }
  float pw[MOEQ_MAX_K];
  float tot = 0.f;
  for (int k = 0; k < p.K; ++k) {
    pw[k] = picked[k] >= 0 ? expf(__ldcg(p.logits + picked[k]) - mx) / z : 0.f;
    tot += pw[k];
  }
  if (lane == 0) {
    for (int k = 0; k < p.K; ++k) {
      const float wk = (p.renorm && tot > 0.f) ? pw[k] / tot : pw[k];
      s_idx[k] = picked[k];
      s_w[k] = wk;
      if (blockIdx.x == 0) {
        if (p.idx_out) p.idx_out[(size_t)l * p.K + k] = forced ? forced[k] : picked[k];
        if (p.w_out) p.w_out[(size_t)l * p.K + k] = wk;
      }
    }
  }
  __syncwarp();
}

// ---- compute pieces ------------------------------------------------------------

// Gate and up rows of one unit from a ring slot; returns h in lane 0.
template <int BITS>
__device__ __forceinline__ float gateup_from_slot(const unsigned char* slot, int H, int G, const uint4* img,
                                                  const float2* tab, float inv_sc) {
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
    const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, img, tab);
    part[0] += chunk_dot_x<BITS>(qg, X, gsb[g], two ? gsb[g + 1] : 0u, two);
    part[1] += chunk_dot_x<BITS>(qu, X, usb[g], two ? usb[g + 1] : 0u, two);
  }
  const float v = transpose_reduce<2>(part);
  const float up = __shfl_sync(0xFFFFFFFFu, v, 16);
  return silu_f(v * inv_sc) * (up * inv_sc);
}

// Adds coef * (4 rows of one down block) into acc (per-lane partials).
template <int BITS>
__device__ __forceinline__ void down_block_acc(const unsigned char* blk, int I, int G, const uint4* img,
                                               const float2* tab, float coef, float (&acc)[kDnBlk]) {
  const int lane = threadIdx.x & 31;
  const int rowb = I * BITS / 8, ng = I / G, nchunk = I * BITS / 128;
  const bool two = (BITS == 2) && (G == 32);
  const uint32_t* sb = reinterpret_cast<const uint32_t*>(blk + kDnBlk * rowb);
  for (int c = lane; c < nchunk; c += 32) {
    const ChunkX<BITS> X = load_chunk_x<BITS>(c, nchunk, img, tab);
    const int g = chunk_group<BITS>(c, G, two);
#pragma unroll
    for (int r = 0; r < kDnBlk; ++r) {
      const uint4 q = *reinterpret_cast<const uint4*>(blk + (size_t)r * rowb + (size_t)c * 16);
      acc[r] += coef * chunk_dot_x<BITS>(q, X, sb[r * ng + g], two ? sb[r * ng + g + 1] : 0u, two);
    }
  }
}

__global__ void __launch_bounds__(kStackThreads, 1) k_decode_layers(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t full_bar[kMaxSlots], empty_bar[kMaxSlots], c_bar[2], cfree_bar;
  __shared__ int s_kind[kMaxSlots], s_a[kMaxSlots], s_b[kMaxSlots], s_last[kMaxSlots];
  __shared__ int s_idx[MOEQ_MAX_K];
  __shared__ float s_w[MOEQ_MAX_K];
  __shared__ float s_part[kMaxRouterRowsPerCta][2];
  __shared__ float s_red[kCWarps][MOEQ_MAX_K + 1];
  __shared__ float s_hsc[MOEQ_MAX_K + 1], s_hinv[MOEQ_MAX_K + 1];
  __shared__ float s_misc[4];  // 0: 2^-e of the x image, 1: gamma, 2: CTA sum of squares
  __shared__ volatile int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int nr = strided_count(c, G, p.E);
  const int nsu = strided_count(c, G, p.I);
  const int nru = strided_count(c, G, p.K * p.I);
  const int nblk = strided_count(c, G, p.H / kDnBlk);
  const int per_layer = 2 * nr + nsu + nru;
  unsigned* sync_count = &p.ctrl->sync_count;

  if (tid == 0) {
    for (int i = 0; i < p.nslot; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      s_last[i] = -1;
    }
    mbar_init(&c_bar[0], 1);
    mbar_init(&c_bar[1], 1);
    mbar_init(&cfree_bar, kCWarps);
    s_abort = 0;
    s_misc[2] = 0.f;
    fence_mbar_init();
  }
  __syncthreads();

  auto fail = [&](void) {
    set_error(p.ctrl, MOE_ERR_TIMEOUT);
    s_abort = 1;
  };

  if (warp == kCWarps) {
    // ===================== producer warp =====================
    Ring R{full_bar, empty_bar, s_kind, s_a, s_b, s_last, sm + p.sm_ring, p.slot_bytes, p.nslot, 0u};
    int c_last[2] = {-1, -1};  // last layer whose down copies were issued, per down barrier
    unsigned char* regc = sm + p.sm_regc;
    issue_pre(p, R, 0, nr, nsu, &s_abort);
    for (int l = 0; l < p.n_layers; ++l) {
      if (l > 0 && !mbar_wait(&cfree_bar, (l - 1) & 1, &s_abort) && lane == 0) fail();
      __syncwarp();
      // shared expert's down blocks (known before routing)
      if (lane == 0 && !s_abort) {
        const uint32_t tot = issue_down_slot(p, regc, p.K, p.L[l].shared, p.off_s, p.bits_s, nblk, &c_bar[0], false);
        mbar_arrive_expect_tx(&c_bar[0], tot);
        issue_down_slot(p, regc, p.K, p.L[l].shared, p.off_s, p.bits_s, nblk, &c_bar[0], true);
        c_last[0] = l;
      }
      // routing
      if (!counter_wait(sync_count, (unsigned)(3 * l + 1) * G, &s_abort) && lane == 0) fail();
      __syncwarp();
      producer_topk(p, l, s_idx, s_w);
      // routed experts' down blocks, then their gate/up units
      if (lane == 0 && !s_abort) {
        uint32_t tot = 0;
        for (int k = 0; k < p.K; ++k)
          if (s_idx[k] >= 0)
            tot += issue_down_slot(p, regc, k, p.L[l].experts + (size_t)s_idx[k] * p.rec_r, p.off_r, p.bits_r, nblk,
                                   &c_bar[1], false);
        mbar_arrive_expect_tx(&c_bar[1], tot);
        for (int k = 0; k < p.K; ++k)
          if (s_idx[k] >= 0)
            issue_down_slot(p, regc, k, p.L[l].experts + (size_t)s_idx[k] * p.rec_r, p.off_r, p.bits_r, nblk,
                            &c_bar[1], true);
        c_last[1] = l;
      }
      __syncwarp();
      issue_routed(p, R, l, nru, s_idx, &s_abort);
      if (l + 1 < p.n_layers) issue_pre(p, R, l + 1, nr, nsu, &s_abort);
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
    const uint4* img4 = reinterpret_cast<const uint4*>(sm + p.sm_img4);
    const float2* tab4 = reinterpret_cast<const float2*>(sm + p.sm_tab4);
    const uint4* img2 = reinterpret_cast<const uint4*>(sm + p.sm_img2);
    const float2* tab2 = reinterpret_cast<const float2*>(sm + p.sm_tab2);
    const unsigned char* ring = sm + p.sm_ring;
    const unsigned char* regc = sm + p.sm_regc;

    for (int l = 0; l < p.n_layers; ++l) {
      // ---- stage x_l ----
      float inv_norm = 1.f;
      if (l > 0) {
        if (tid == 0 && !counter_wait(sync_count, (unsigned)(3 * l) * G, &s_abort)) fail();
        named_sync(1, kCThreads);
        inv_norm = rsqrtf(__ldcg(p.ss + (l - 1)) / (float)H + p.eps);
      }
      float amax = 0.f, gdot = 0.f;
      const uint16_t* gw = p.L[l].gate_w;
      for (int j = tid; j < H; j += kCThreads) {
        uint16_t xb;
        if (l == 0)
          xb = p.x_in[j];
        else
          xb = f32_to_bf16_bits(__ldcg(p.r + j) * inv_norm);
        xs[j] = xb;
        const float xf = bf16_bits_to_f32(xb);
        amax = fmaxf(amax, fabsf(xf));
        if (gw) gdot += bf16_bits_to_f32(gw[j]) * xf;
      }
      amax = warp_max(amax);
      gdot = warp_sum(gdot);
      if (lane == 0) {
        s_red[warp][0] = amax;
        s_red[warp][1] = gdot;
      }
      named_sync(1, kCThreads);
      if (tid == 0) {
        float m = 0.f, d = 0.f;
        for (int w = 0; w < kCWarps; ++w) {
          m = fmaxf(m, s_red[w][0]);
          d += s_red[w][1];
        }
        const int ex = fp16_scale_exp(m);
        s_misc[0] = pow2f(ex);
        s_misc[1] = gw ? 1.f / (1.f + expf(-d)) : 1.f;
        s_misc[3] = pow2f(-ex);
      }
      named_sync(1, kCThreads);
      {
        const float sc = s_misc[0];
        auto get = [&](int j) { return bf16_bits_to_f32(xs[j]); };
        if (p.need4)
          stage_image<4>(get, H, sc, reinterpret_cast<__half*>(sm + p.sm_img4), reinterpret_cast<float2*>(sm + p.sm_tab4),
                         tid, kCThreads);
        if (p.need2)
          stage_image<2>(get, H, sc, reinterpret_cast<__half*>(sm + p.sm_img2), reinterpret_cast<float2*>(sm + p.sm_tab2),
                         tid, kCThreads);
      }
      named_sync(1, kCThreads);
      const float x_inv = s_misc[3];

      // ---- ring items: router half-rows, then gate/up units ----
      const int base = l * per_layer;
      bool router_synced = false;
      auto router_barrier = [&](void) {
        if (warp == 0) {
          named_sync(2, kCThreads);
          if (lane == 0) {
            for (int m = 0; m < nr; ++m) __stcg(p.logits + c + G * m, s_part[m][0] + s_part[m][1]);
            __threadfence();
            atomicAdd(sync_count, 1u);
          }
          __syncwarp();
        } else {
          named_arrive(2, kCThreads);
        }
      };
      for (int j = base + warp; j < base + per_layer; j += kCWarps) {
        if (!router_synced && j >= base + 2 * nr) {
          router_barrier();
          router_synced = true;
        }
        const int slot = j % p.nslot;
        const bool ok = mbar_wait(&full_bar[slot], (j / p.nslot) & 1, &s_abort);
        if (!ok && lane == 0 && !s_abort) fail();
        if (ok) {
          const int kind = s_kind[slot], a = s_a[slot], b = s_b[slot];
          const unsigned char* sl = ring + (size_t)slot * p.slot_bytes;
          if (kind == kItemRouterHalf) {
            const int nv = H / 16;  // 16-byte words in a half row
            const uint4* wv = reinterpret_cast<const uint4*>(sl);
            const uint4* xv = reinterpret_cast<const uint4*>(xs + b * (H / 2));
            float acc = 0.f;
            for (int v = lane; v < nv; v += 32) acc = dot8_bf16(wv[v], xv[v], acc);
            acc = warp_sum(acc);
            if (lane == 0) s_part[a][b] = acc;
          } else {
            float hv = 0.f;
            if (kind == kItemGateUp) {
              const int bits = a < K ? p.bits_r : p.bits_s;
              hv = bits == 4 ? gateup_from_slot<4>(sl, H, p.G, img4, tab4, x_inv)
                             : gateup_from_slot<2>(sl, H, p.G, img2, tab2, x_inv);
            }
            if (lane == 0) __stcg(p.h + (size_t)a * I + b, hv);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
      }
      if (!router_synced) router_barrier();

      // ---- sync 2: h complete ----
      named_sync(1, kCThreads);
      if (tid == 0) {
        __threadfence();
        atomicAdd(sync_count, 1u);
        if (!counter_wait(sync_count, (unsigned)(3 * l + 2) * G, &s_abort)) fail();
      }
      named_sync(1, kCThreads);

      // ---- stage h images (one per slot) ----
      {
        float am[MOEQ_MAX_K + 1];
#pragma unroll
        for (int k = 0; k <= MOEQ_MAX_K; ++k) am[k] = 0.f;
        for (int j = tid; j < I; j += kCThreads) {
#pragma unroll
          for (int k = 0; k <= MOEQ_MAX_K; ++k)
            if (k <= K) am[k] = fmaxf(am[k], fabsf(__ldcg(p.h + (size_t)k * I + j)));
        }
#pragma unroll
        for (int k = 0; k <= MOEQ_MAX_K; ++k) {
          const float m = warp_max(am[k]);
          if (lane == 0 && k <= K) s_red[warp][k] = m;
        }
        named_sync(1, kCThreads);
        if (tid <= K) {
          float m = 0.f;
          for (int w = 0; w < kCWarps; ++w) m = fmaxf(m, s_red[w][tid]);
          const int ex = fp16_scale_exp(m);
          s_hsc[tid] = pow2f(ex);
          s_hinv[tid] = pow2f(-ex);
        }
        named_sync(1, kCThreads);
        for (int k = 0; k <= K; ++k) {
          const float* hk = p.h + (size_t)k * I;
          auto get = [&](int j) { return __ldcg(hk + j); };
          __half* img = reinterpret_cast<__half*>(sm + p.sm_himg + (size_t)k * p.himg_stride);
          float2* tab = reinterpret_cast<float2*>(sm + p.sm_htab + (size_t)k * p.htab_stride);
          if ((k < K ? p.bits_r : p.bits_s) == 4)
            stage_image<4>(get, I, s_hsc[k], img, tab, tid, kCThreads);
          else
            stage_image<2>(get, I, s_hsc[k], img, tab, tid, kCThreads);
        }
        named_sync(1, kCThreads);
      }

      // ---- down + combine for this CTA's row blocks ----
      const bool ok0 = mbar_wait(&c_bar[0], l & 1, &s_abort);
      const bool ok1 = mbar_wait(&c_bar[1], l & 1, &s_abort);
      if (!(ok0 && ok1) && tid == 0 && !s_abort) fail();
      const float gamma = s_misc[1];
      float ssq = 0.f;
      for (int m = warp; m < nblk; m += kCWarps) {
        const int i0 = (c + G * m) * kDnBlk;
        float acc[kDnBlk] = {0.f, 0.f, 0.f, 0.f};
        if (!s_abort) {
          for (int k = 0; k <= K; ++k) {
            const float wk = k < K ? (s_idx[k] >= 0 ? s_w[k] : 0.f) : gamma;
            if (wk == 0.f) continue;
            const float coef = wk * s_hinv[k];
            const unsigned char* blk = regc + ((size_t)k * p.nblk_max + m) * p.dblk_bytes;
            const uint4* img = reinterpret_cast<const uint4*>(sm + p.sm_himg + (size_t)k * p.himg_stride);
            const float2* tab = reinterpret_cast<const float2*>(sm + p.sm_htab + (size_t)k * p.htab_stride);
            if ((k < K ? p.bits_r : p.bits_s) == 4)
              down_block_acc<4>(blk, I, p.G, img, tab, coef, acc);
            else
              down_block_acc<2>(blk, I, p.G, img, tab, coef, acc);
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
        __threadfence();
        atomicAdd(sync_count, 1u);
      }
    }

    // ---- optional RMSNorm'd bf16 output of the last layer ----
    if (p.xnorm_out) {
      if (tid == 0 && !counter_wait(sync_count, (unsigned)(3 * p.n_layers) * G, &s_abort)) fail();
      named_sync(1, kCThreads);
      const float inv = rsqrtf(__ldcg(p.ss + (p.n_layers - 1)) / (float)H + p.eps);
      for (int t = tid; t < nblk * kDnBlk; t += kCThreads) {
        const int i = (c + G * (t / kDnBlk)) * kDnBlk + (t % kDnBlk);
        p.xnorm_out[i] = f32_to_bf16_bits(p.resid_out[i] * inv);
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
