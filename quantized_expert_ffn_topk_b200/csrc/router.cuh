// router.cuh -- moe_router_topk: router GEMV (bf16 weights and input, fp32
// accumulation), then softmax and top-K done by the last CTA to finish.
#pragma once

#include "common.cuh"

namespace moeq {

#ifndef MOEQ_ROUTER_WARPS
#define MOEQ_ROUTER_WARPS 8
#endif
constexpr int kRouterWarps = MOEQ_ROUTER_WARPS;  // warps per CTA, one expert row per warp at a time
constexpr int kRouterTokTile = 8;   // tokens of one CTA (its x staged in shared memory)
constexpr int kRouterUnroll = 8;    // 16-byte loads of one row in flight per lane (the rows were prefetched to L2)
constexpr int kRouterMaxE = 1024;   // experts the selection holds: 32 keys per lane

struct RouterParams {
  const uint16_t* x;       // [B, H] bf16
  const uint16_t* wr;      // [E, H] bf16
  const int32_t* forced;   // [B, K] or null
  int32_t* idx;            // [B, K]
  float* w;                // [B, K]
  float* logits;           // [B, E] (workspace or caller buffer)
  WsCtrl* ctrl;
  int B, H, E, K, renorm;
};

// Eight bf16 (one 16-byte word) against eight staged x values.
__device__ __forceinline__ float dot8_bf16(uint4 wv, const uint4 xv, float acc) {
  const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
  const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc = fmaf(__uint_as_float(ww[i] << 16), __uint_as_float(xx[i] << 16), acc);
    acc = fmaf(__uint_as_float(ww[i] & 0xFFFF0000u), __uint_as_float(xx[i] & 0xFFFF0000u), acc);
  }
  return acc;
}

// Order-preserving key of a logit (NaN read as -inf): a larger value has a
// larger key, -0 ranks as +0, and key 0 lies below every value ("taken").
constexpr uint32_t kKeyNegInf = 0x007FFFFFu;  // the key of -inf
__device__ __forceinline__ uint32_t logit_key(float v) {
  uint32_t u = __float_as_uint(v == v ? v : -INFINITY);
  u = u == 0x80000000u ? 0u : u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Top-K of one token's logits (E <= 32 * NV) by one warp, softmax weights at
// the picks (router gating of the Flash-MoE page, "Metal Compute Shaders").
// Lane l keeps the keys of logits l + 32 j in registers; each of the K rounds
// takes a warp-wide max over the keys and a warp-wide min over the indices
// holding it (ties go to the lower index), and the owner lane clears its key.
template <int NV>
__device__ void topk_one_token_nv(const float* lg, int E, int K, int renorm, const int32_t* forced, int32_t* idx_out,
                                  float* w_out, WsCtrl* ctrl) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NV];
  uint32_t lk = 0u;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    const int e = lane + 32 * j;
    key[j] = e < E ? logit_key(lg[e]) : 0u;
    lk = max(lk, key[j]);
  }
  const uint32_t m0 = __reduce_max_sync(0xFFFFFFFFu, lk);
  const float mx = m0 > kKeyNegInf ? key_logit(m0) : -INFINITY;
  float z = 0.f;
  for (int e = lane; e < E; e += 32) z += expf(lg[e] - mx);
  z = warp_sum(z);
  int picked[MOEQ_MAX_K];
  if (forced) {
    for (int k = 0; k < K; ++k) {
      int e = forced[k];
      if (e < 0 || e >= E) {
        if (lane == 0) set_error(ctrl, MOE_ERR_INDEX);
        e = -1;
      }
      picked[k] = e;
    }
  } else {
    for (int k = 0; k < K; ++k) {
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, lk);
      uint32_t cand = 0xFFFFFFFFu;
#pragma unroll
      for (int j = NV - 1; j >= 0; --j) cand = key[j] == m ? (uint32_t)(lane + 32 * j) : cand;
      const uint32_t bi = __reduce_min_sync(0xFFFFFFFFu, cand);
      if ((bi & 31u) == (uint32_t)lane) {
        lk = 0u;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
          key[j] = j == (int)(bi >> 5) ? 0u : key[j];
          lk = max(lk, key[j]);
        }
      }
      if (m > kKeyNegInf) {
        picked[k] = (int)bi;
      } else {  // no finite logit left (NaN input): no expert
        if (lane == 0) set_error(ctrl, MOE_ERR_INDEX);
        picked[k] = -1;
      }
    }
  }
  float p[MOEQ_MAX_K];
  float tot = 0.f;
  for (int k = 0; k < K; ++k) {
    p[k] = picked[k] >= 0 ? expf(lg[picked[k]] - mx) / z : 0.f;
    tot += p[k];
  }
  if (lane == 0) {
    for (int k = 0; k < K; ++k) {
      idx_out[k] = forced ? forced[k] : picked[k];
      w_out[k] = (renorm && tot > 0.f) ? p[k] / tot : p[k];
    }
  }
}

// Softmax and top-K of one token's logits `lg` (shared memory) by NW warps
// together (threads 0 .. 32*NW-1, each holding up to PT logits: E <= 32*NW*PT)
// (router gating as the Flash-MoE page gives it in "Metal Compute Shaders":
// softmax over all experts, the K largest, weights renormalised on request).
// Thread t holds logits t + 32*NW*i as order-preserving keys; each warp takes
// its K best by K rounds of a warp-wide max over the keys and a warp-wide min
// over the indices holding it (ties go to the lower index), and warp 0 takes
// the K best of the warps' candidates the same way: the top K of all logits
// are among the warps' top K, so the picks are those of one global ranking.
// The normaliser is summed per warp around the warp's own maximum and
// rescaled to the global one. `sync` is the barrier of the NW warps. Warp 0's
// lanes k < K end with sel[k] (the pick; -1 for none: no finite logit left or
// an invalid forced index) and wsel[k] (its weight) written; the other warps
// return after the barrier.
template <int NW>
struct SelScratch {
  uint32_t key[NW * MOEQ_MAX_K];  // warp w's K best at w*K .. w*K+K-1, in rank order
  uint32_t idx[NW * MOEQ_MAX_K];
  float m[NW], z[NW];            // each warp's max logit and sum of exp(v - max)
};

template <int NW, int PT, typename Sync>
__device__ void block_select(const float* lg, int E, int K, int renorm, const int32_t* forced, SelScratch<NW>& S,
                             Sync sync, int* sel, float* wsel, WsCtrl* ctrl) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kT = NW * 32;
  uint32_t key[PT];
  uint32_t kmax = 0u;
#pragma unroll
  for (int i = 0; i < PT; ++i) {
    const int e = tid + kT * i;
    key[i] = e < E ? logit_key(lg[e]) : 0u;
    kmax = max(kmax, key[i]);
  }
  const uint32_t wm = __reduce_max_sync(0xFFFFFFFFu, kmax);
  const float mw = wm > kKeyNegInf ? key_logit(wm) : -INFINITY;
  float zw = 0.f;
  if (mw > -INFINITY) {  // warp-uniform
#pragma unroll
    for (int i = 0; i < PT; ++i) zw += key[i] > kKeyNegInf ? __expf(key_logit(key[i]) - mw) : 0.f;
    zw = warp_sum(zw);
  }
  if (!forced) {
    uint32_t ck = 0u;
    int ci = -1;
#pragma unroll 1
    for (int kk = 0; kk < K; ++kk) {
      uint32_t km = 0u;
#pragma unroll
      for (int i = 0; i < PT; ++i) km = max(km, key[i]);
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, km);
      uint32_t cand = 0xFFFFFFFFu;
#pragma unroll
      for (int i = PT - 1; i >= 0; --i) cand = key[i] == m ? (uint32_t)(tid + kT * i) : cand;
      const uint32_t bi = __reduce_min_sync(0xFFFFFFFFu, cand);
#pragma unroll
      for (int i = 0; i < PT; ++i) key[i] = bi == (uint32_t)(tid + kT * i) ? 0u : key[i];
      if (lane == kk) {
        ck = m;
        ci = (int)bi;
      }
    }
    if (lane < K) {
      S.key[warp * K + lane] = ck;
      S.idx[warp * K + lane] = (uint32_t)ci;
    }
  }
  if (lane == 0) {
    S.m[warp] = mw;
    S.z[warp] = zw;
  }
  sync();
  if (warp != 0) return;

  float mx = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) mx = fmaxf(mx, S.m[w]);
  float z = (lane < NW && S.m[lane] > -INFINITY) ? S.z[lane] * __expf(S.m[lane] - mx) : 0.f;
  z = warp_sum(z);
  int pick_e = -1;     // lane k (< K) ends up holding pick k
  float pick_l = 0.f;  // and its logit
  if (forced) {
    if (lane < K) {
      const int bi = forced[lane];
      const bool okf = bi >= 0 && bi < E;
      pick_e = okf ? bi : -1;
      pick_l = okf ? lg[bi] : -INFINITY;
    }
  } else {
    // candidate c = lane + 32 j of the warps' NW * K
    constexpr int NC = (NW * MOEQ_MAX_K + 31) / 32;
    const int nc = NW * K;
    uint32_t ck[NC];
    uint32_t ci[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int c = lane + 32 * j;
      ck[j] = c < nc ? S.key[c] : 0u;
      ci[j] = c < nc ? S.idx[c] : 0xFFFFFFFFu;
    }
#pragma unroll 1
    for (int kk = 0; kk < K; ++kk) {
      uint32_t km = 0u;
#pragma unroll
      for (int j = 0; j < NC; ++j) km = max(km, ck[j]);
      const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, km);
      uint32_t cand = 0xFFFFFFFFu;
#pragma unroll
      for (int j = 0; j < NC; ++j) cand = ck[j] == m ? min(cand, ci[j]) : cand;
      const uint32_t bi = __reduce_min_sync(0xFFFFFFFFu, cand);
#pragma unroll
      for (int j = 0; j < NC; ++j) ck[j] = (ck[j] == m && ci[j] == bi) ? 0u : ck[j];
      if (lane == kk) {
        const bool fin = m > kKeyNegInf;  // no finite logit left: no expert
        pick_e = fin ? (int)bi : -1;
        pick_l = fin ? key_logit(m) : -INFINITY;
      }
    }
  }
  if (lane < K && pick_e < 0) set_error(ctrl, MOE_ERR_INDEX);
  const float pw = (lane < K && pick_e >= 0) ? __expf(pick_l - mx) / z : 0.f;
  const float tot = warp_sum(pw);
  if (lane < K) {
    sel[lane] = pick_e;
    wsel[lane] = (renorm && tot > 0.f) ? pw / tot : pw;
  }
}

// E <= 512 keeps 16 keys per lane, else 32.
__device__ __forceinline__ void topk_one_token(const float* lg, int E, int K, int renorm, const int32_t* forced,
                                               int32_t* idx_out, float* w_out, WsCtrl* ctrl) {
  if (E <= 512) topk_one_token_nv<16>(lg, E, K, renorm, forced, idx_out, w_out, ctrl);
  else topk_one_token_nv<kRouterMaxE / 32>(lg, E, K, renorm, forced, idx_out, w_out, ctrl);
}

// grid (E/kRouterWarps, ceil(B/kRouterTokTile)): CTA (c, j) dots rows of
// warps c*kRouterWarps.. with tokens 8j..8j+7; the last CTA of column j to
// finish selects for those tokens.
// TT: tokens of a CTA's tile (kRouterTokTile, or 1 for a single token: then
// one accumulator, and all of a row's 16-byte loads in flight at once).
template <int TT>
__global__ void __launch_bounds__(kRouterWarps * 32, 1) k_router_topk(RouterParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);  // [tok_tile, H]
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t s_bar;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gwarp = blockIdx.x * kRouterWarps + warp, nwarps = gridDim.x * kRouterWarps;
  const int nvec = p.H / 8;  // 16-byte words per row
  const int b0 = blockIdx.y * TT, tb = min(TT, p.B - b0);
  constexpr int UNR = TT == 1 ? 2 * kRouterUnroll : kRouterUnroll;  // loads of a row in flight per lane

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
  }
  pdl_trigger();
  // the weight rows do not depend on the previous kernel: pull them into L2
  if (lane == 0 && blockIdx.y == 0)
    for (int e = gwarp; e < p.E; e += nwarps) prefetch_l2(p.wr + (size_t)e * p.H, (uint32_t)p.H * 2);
  __syncthreads();
  pdl_wait();
  // the token tile's x rows (contiguous) in one bulk copy; bounded wait (one
  // token reads its x at L2 beside each row's loads instead: no wait first)
  if (TT > 1) {
    if (threadIdx.x == 0) {
      const uint32_t bytes = (uint32_t)tb * (uint32_t)p.H * 2u;
      mbar_arrive_expect_tx(&s_bar, bytes);
      bulk_g2s(xs, p.x + (size_t)b0 * p.H, bytes, &s_bar);
    }
    const long long budget = wait_budget(p.ctrl);
    const long long t0 = clock64();
    bool ok;
    while (!(ok = mbar_try_wait(&s_bar, 0u)) && clock64() - t0 < budget) __nanosleep(32);
    if (!ok && threadIdx.x == 0) set_error(p.ctrl, MOE_ERR_TIMEOUT);
    __syncthreads();
  }
  const uint4* x1 = reinterpret_cast<const uint4*>(p.x + (size_t)b0 * p.H);
  for (int e = gwarp; e < p.E; e += nwarps) {
    const uint16_t* row = p.wr + (size_t)e * p.H;
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.f;
    for (int v0 = lane; v0 < nvec; v0 += 32 * UNR) {
      uint4 wv[UNR], xv[TT == 1 ? UNR : 1];
#pragma unroll
      for (int u = 0; u < UNR; ++u)
        if (v0 + 32 * u < nvec) {
          wv[u] = ld_stream16(row + (size_t)(v0 + 32 * u) * 8);
          if constexpr (TT == 1) xv[u] = __ldcg(x1 + v0 + 32 * u);
        }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int v = v0 + 32 * u;
        if (v < nvec) {
          if constexpr (TT == 1) {
            acc[0] = dot8_bf16(wv[u], xv[u], acc[0]);
          } else {
#pragma unroll
            for (int t = 0; t < TT; ++t)
              if (t < tb) acc[t] = dot8_bf16(wv[u], reinterpret_cast<const uint4*>(xs + (size_t)t * p.H)[v], acc[t]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t < tb) {
        float sum = warp_sum(acc[t]);
        if (lane == 0) p.logits[(size_t)(b0 + t) * p.E + e] = sum;
      }
    }
  }
  // The last CTA of this token tile to arrive selects for its tokens. The
  // ticket is one acquire-release add: it publishes this CTA's logits (stored
  // before the barrier) and, for the last CTA, orders its reads of every
  // other CTA's logits after their adds.
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned t;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(t) : "l"(&p.ctrl->router_ticket[blockIdx.y])
                 : "memory");
    s_last = (t == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  float* lsm = reinterpret_cast<float*>(smem_raw);  // this tile's logits
  {
    // every load of the tile in flight before the stores (the logits come from L2)
    const float* src = p.logits + (size_t)b0 * p.E;
    const int n = tb * p.E;
    for (int i0 = 0; i0 < n; i0 += 8 * (int)blockDim.x) {
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * (int)blockDim.x + (int)threadIdx.x;
        v[j] = i < n ? __ldcg(src + i) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * (int)blockDim.x + (int)threadIdx.x;
        if (i < n) lsm[i] = v[j];
      }
    }
  }
  __syncthreads();
  if (tb == 1) {
    // one token: all warps select together (a warp alone would walk E/32
    // keys per lane through K rounds)
    __shared__ SelScratch<kRouterWarps> S;
    const int32_t* forced = p.forced ? p.forced + (size_t)b0 * p.K : nullptr;
    block_select<kRouterWarps, kRouterMaxE / (32 * kRouterWarps)>(lsm, p.E, p.K, p.renorm, forced, S,
                                                                  [] { __syncthreads(); }, p.idx + (size_t)b0 * p.K,
                                                                  p.w + (size_t)b0 * p.K, p.ctrl);
    if (forced && warp == 0 && lane < p.K) p.idx[(size_t)b0 * p.K + lane] = forced[lane];
  } else {
    for (int t = warp; t < tb; t += kRouterWarps) {
      const int b = b0 + t;
      topk_one_token(lsm + (size_t)t * p.E, p.E, p.K, p.renorm, p.forced ? p.forced + (size_t)b * p.K : nullptr,
                     p.idx + (size_t)b * p.K, p.w + (size_t)b * p.K, p.ctrl);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) p.ctrl->router_ticket[blockIdx.y] = 0u;
}

}  // namespace moeq
