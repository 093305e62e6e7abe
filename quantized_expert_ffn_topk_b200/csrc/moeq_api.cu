// moeq_api.cu -- host side of libmoeq.so: argument checks, launch shapes and
// the extern "C" entry points declared in include/moeq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "combine.cuh"
#include "common.cuh"
#include "ffn.cuh"
#include "grouped.cuh"
#include "pack.cuh"
#include "router.cuh"
#include "stack.cuh"

namespace moeq {
namespace {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool bits_ok(int bits) { return bits >= 2 && bits <= 4; }
inline bool group_ok(int g) { return g == 32 || g == 64 || g == 128; }

// A row of `cols` codes must be whole 16-byte chunks and whole groups.
inline bool cols_ok(int cols, int bits, int group) {
  return cols > 0 && cols % group == 0 && ((int64_t)cols * bits) % 128 == 0;
}

inline moe_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int g_num_sms = 0;
inline int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 148;
    g_num_sms = n > 0 ? n : 148;
  }
  return g_num_sms;
}

// Launch with programmatic dependent launch allowed, so a kernel's prologue
// may overlap the tail of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
moe_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// Raise a kernel's dynamic shared-memory limit to `bytes` once per (kernel,
// device): the attribute is set only when a call needs more than before.
template <typename K>
moe_status ensure_smem(K kern, size_t bytes) {
  if (bytes <= 48 * 1024) return MOE_OK;
  if (bytes > 227 * 1024) return MOE_ERR_UNSUPPORTED;
  struct Seen { const void* fn; int dev; size_t bytes; };
  static std::mutex mu;
  static Seen seen[64];
  static int nseen = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(mu);
  Seen* e = nullptr;
  for (int i = 0; i < nseen; ++i)
    if (seen[i].fn == fn && seen[i].dev == dev) e = &seen[i];
  if (e && e->bytes >= bytes) return MOE_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (e) e->bytes = bytes;
  else if (nseen < 64) seen[nseen++] = Seen{fn, dev, bytes};
  return MOE_OK;
}

// Workspace layout: [control 256 B][logits B*E fp32][h B*(K+1)*I fp32]
//                   [r B*H fp32][ss kStackMaxCtas fp32: partial sums of squares]
//                   [token grouping][input images]
struct WsLayout {
  size_t logits, h, r, ss;
  size_t cnt, off, list, act, nact;  // token grouping (batches)
  size_t ximg, himg;                 // per-token input images (batches)
  int ximg_stride, ximg_gs, himg_stride, himg_gs;
  size_t total;
};
inline WsLayout ws_layout(int B, int K, int H, int I, int E) {
  WsLayout l{};
  size_t o = sizeof(WsCtrl);
  l.logits = o;
  o += align_up((size_t)B * E * sizeof(float));
  l.h = o;
  o += align_up((size_t)B * (K + 1) * I * sizeof(float));
  l.r = o;
  o += align_up((size_t)B * H * sizeof(float));
  l.ss = o;
  o += align_up((size_t)kStackMaxCtas * sizeof(float));
  l.cnt = o;
  o += align_up((size_t)E * 4);
  l.off = o;
  o += align_up((size_t)(E + 1) * 4);
  l.list = o;
  o += align_up((size_t)B * K * 4);
  l.act = o;
  o += align_up((size_t)(E + kGrpExtraChunks) * 3 * 4);
  l.nact = o;
  o += align_up(3 * 4);  // chunks, then the two grouped kernels' unit counters
  // images: planes then (scale, sum) per group; the smallest group (32) sizes them
  l.ximg_gs = (int)align_up(qimg_plane_bytes(H), 16);
  l.ximg_stride = (int)align_up(l.ximg_gs + qimg_gs_bytes(H, 32), 256);
  l.himg_gs = (int)align_up(qimg_plane_bytes(I), 16);
  l.himg_stride = (int)align_up(l.himg_gs + qimg_gs_bytes(I, 32), 256);
  l.ximg = o;
  o += (size_t)B * l.ximg_stride;
  l.himg = o;
  o += (size_t)B * (K + 1) * l.himg_stride;
  l.total = o;
  return l;
}

moe_status check_layer(const moe_layer_q* L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (L->H <= 0 || L->I <= 0 || L->E <= 0 || L->K <= 0) return MOE_ERR_INVALID_ARG;
  if (L->K > MOEQ_MAX_K || L->K > L->E) return MOE_ERR_INVALID_ARG;
  if (!bits_ok(L->bits_routed) || !bits_ok(L->bits_shared) || !group_ok(L->group)) return MOE_ERR_UNSUPPORTED;
  for (int bits : {L->bits_routed, L->bits_shared})
    if (moe_expert_bytes(L->H, L->I, bits, L->group) == 0) return MOE_ERR_UNSUPPORTED;
  if (!L->experts || !L->shared || !L->router_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(L->experts) || !aligned16(L->shared) || !aligned16(L->router_w)) return MOE_ERR_ALIGN;
  if (L->shared_gate_w && !aligned16(L->shared_gate_w)) return MOE_ERR_ALIGN;
  return MOE_OK;
}

bool ffn_plan(FfnParams& p, int G, size_t& gu_bytes, size_t& dn_bytes);  // below

// The grouped kernels' instances: one format compiled in when the routed and
// shared widths agree, else the instances that pick the format per item.
struct GrpKernels {
  void (*gate_up)(GrpParams);
  void (*down)(GrpParams);
};
GrpKernels grp_kernels(int br, int bs, int G) {
#define MOEQ_GRP_CASE(B, Gp, KS) \
  if (br == B && bs == B && G == Gp) return GrpKernels{k_ffn_grp<false, B, KS>, k_ffn_grp<true, B, KS>};
  MOEQ_GRP_CASE(4, 32, 1)
  MOEQ_GRP_CASE(4, 64, 2)
  MOEQ_GRP_CASE(4, 128, 4)
  MOEQ_GRP_CASE(2, 32, 1)
  MOEQ_GRP_CASE(2, 64, 2)
  MOEQ_GRP_CASE(2, 128, 4)
  MOEQ_GRP_CASE(3, 64, 2)
  MOEQ_GRP_CASE(3, 128, 4)
#undef MOEQ_GRP_CASE
  return GrpKernels{k_ffn_grp<false, 0, 0>, k_ffn_grp<true, 0, 0>};
}


// The one-token FFN kernels' dot: the tensor-core dot, or with
// MOEQ_BATCH1_DOT=fma in the environment the fp32 CUDA-core dot (a switch
// for comparing the two on the same kernels; read once).
int batch1_dot_fma() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MOEQ_BATCH1_DOT");
    v = (e && strcmp(e, "fma") == 0) ? 1 : 0;
  }
  return v;
}

__global__ void k_ws_debug(WsCtrl* c, unsigned wait_us, int withhold_cta) {
  c->wait_us = wait_us;
  c->withhold_cta = withhold_cta;
}

}  // namespace

// Arguments of moe_expert_ffn_q other than the workspace (layer, pointers,
// batch, alignment); MOE_OK or the status the call returns.
moe_status ffn_check_args(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx, const float* y_out) {
  moe_status st = check_layer(L);
  if (st != MOE_OK) return st;
  if (!x_bf16 || !idx || !y_out) return MOE_ERR_INVALID_ARG;
  if (B <= 0 || B > MOEQ_MAX_B) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(y_out) || !aligned16(idx)) return MOE_ERR_ALIGN;
  return MOE_OK;
}

}  // namespace moeq

using namespace moeq;

extern "C" {

int moe_abi_version(void) { return MOEQ_ABI_VERSION; }

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case MOE_ERR_UNSUPPORTED: return "unsupported bits/group/shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_INDEX: return "expert index out of range (device)";
    case MOE_ERR_TIMEOUT: return "bounded wait timed out (device)";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_RANGE: return "code does not fit its bit width (device)";
  }
  return "unknown status";
}

size_t moe_expert_bytes(int H, int I, int bits, int group) {
  if (H <= 0 || I <= 0 || !bits_ok(bits) || !group_ok(group)) return 0;
  if (bits == 3 && group < 64) return 0;  // a 3-bit block pairs k-steps: group 64 or 128
  if (!cols_ok(H, bits, group) || !cols_ok(I, bits, group)) return 0;
  if (H % kTileRows != 0 || I % 8 != 0) return 0;  // whole tiles of 16 rows
  const size_t hi = 3 * (size_t)H * I;
  return hi * bits / 8 + hi / group * 4;
}

moe_status moe_expert_layout(int H, int I, int bits, int group, size_t lay[6]) {
  if (!lay) return MOE_ERR_INVALID_ARG;
  if (moe_expert_bytes(H, I, bits, group) == 0) return MOE_ERR_UNSUPPORTED;
  const RecGeom g = rec_geom(H, I, bits, group);
  lay[0] = g.U;
  lay[1] = (size_t)g.down_off;
  lay[2] = g.D;
  lay[3] = kTileRows;
  lay[4] = g.blk;
  lay[5] = (size_t)(I / 8);
  return MOE_OK;
}

size_t moe_workspace_bytes(int B, int K, int H, int I, int E) {
  if (B <= 0 || K <= 0 || H <= 0 || I <= 0 || E <= 0) return 0;
  return ws_layout(B, K, H, I, E).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < sizeof(WsCtrl)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGN;
  if (cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

moe_status moe_workspace_debug(void* ws, size_t ws_bytes, unsigned wait_budget_us, int withhold_cta, void* stream) {
  if (!ws || ws_bytes < sizeof(WsCtrl)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGN;
  if (withhold_cta < 0) return MOE_ERR_INVALID_ARG;
  k_ws_debug<<<1, 1, 0, (cudaStream_t)stream>>>(reinterpret_cast<WsCtrl*>(ws), wait_budget_us, withhold_cta);
  return launch_status();
}

moe_status moe_rmsnorm(const float* r, const void* weight_bf16, int B, int H, float eps, void* xnorm_bf16_out,
                       void* stream) {
  if (!r || !xnorm_bf16_out) return MOE_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(r) || !aligned16(xnorm_bf16_out) || (weight_bf16 && !aligned16(weight_bf16))) return MOE_ERR_ALIGN;
  return launch_pdl(k_rmsnorm, dim3(B), dim3(kCombineThreads), 0, (cudaStream_t)stream, r,
                    reinterpret_cast<const uint16_t*>(weight_bf16), H, eps,
                    reinterpret_cast<uint16_t*>(xnorm_bf16_out));
}

moe_status moe_pack_q(const uint8_t* codes, const void* scale_bf16, const void* bias_bf16, int rows, int cols,
                      int bits, int group, void* packed_out, void* sb_out, void* ws, void* stream) {
  if (!codes || !scale_bf16 || !bias_bf16 || !packed_out || !sb_out) return MOE_ERR_INVALID_ARG;
  if (rows < 0) return MOE_ERR_INVALID_ARG;
  if (!bits_ok(bits) || !group_ok(group) || !cols_ok(cols, bits, group)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(codes) || !aligned16(packed_out) || !aligned16(sb_out) || !aligned16(scale_bf16) ||
      !aligned16(bias_bf16) || (ws && !aligned16(ws)))
    return MOE_ERR_ALIGN;
  if (rows == 0) return MOE_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t nchunks = bits == 3 ? (int64_t)rows * cols / 128 : (int64_t)rows * cols * bits / 128;
  const int64_t nsb = (int64_t)rows * (cols / group);
  const unsigned maxg = (unsigned)num_sms() * 8;
  unsigned g1 = (unsigned)std::min<int64_t>((nchunks + 255) / 256, maxg);
  unsigned g2 = (unsigned)std::min<int64_t>((nsb + 255) / 256, maxg);
  WsCtrl* ctrl = reinterpret_cast<WsCtrl*>(ws);
  const size_t rowb = (size_t)cols * bits / 8, sbb = (size_t)(cols / group) * 4;
  const RowPlace pc{reinterpret_cast<unsigned char*>(packed_out), rows, rowb, rowb * rows};
  const RowPlace ps{reinterpret_cast<unsigned char*>(sb_out), rows, sbb, sbb * rows};
  const int cpr = (int)(rowb / 16);
  if (bits == 4)
    k_pack_codes<4><<<g1, 256, 0, s>>>(codes, nchunks, cpr, pc, ctrl);
  else if (bits == 3)
    k_pack_codes3<<<g1, 256, 0, s>>>(codes, nchunks, cols / 128, pc, ctrl);
  else
    k_pack_codes<2><<<g1, 256, 0, s>>>(codes, nchunks, cpr, pc, ctrl);
  k_pack_sb<<<g2, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(scale_bf16), reinterpret_cast<const uint16_t*>(bias_bf16),
                               nsb, cols / group, ps);
  return launch_status();
}

moe_status moe_quantize(const void* w, int in_bf16, int rows, int cols, int bits, int group, uint8_t* codes_out,
                        void* scale_bf16_out, void* bias_bf16_out, void* ws, void* stream) {
  if (!w || !codes_out || !scale_bf16_out || !bias_bf16_out) return MOE_ERR_INVALID_ARG;
  if (rows < 0 || cols <= 0 || (in_bf16 != 0 && in_bf16 != 1)) return MOE_ERR_INVALID_ARG;
  if (!bits_ok(bits) || !group_ok(group) || cols % group != 0) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(w) || !aligned16(codes_out) || !aligned16(scale_bf16_out) || !aligned16(bias_bf16_out) ||
      (ws && !aligned16(ws)))
    return MOE_ERR_ALIGN;
  if (rows == 0) return MOE_OK;
  const int64_t ngroups = (int64_t)rows * (cols / group);
  const unsigned grid = (unsigned)std::min<int64_t>((ngroups + 7) / 8, (int64_t)num_sms() * 16);
  cudaStream_t s = (cudaStream_t)stream;
  WsCtrl* ctrl = reinterpret_cast<WsCtrl*>(ws);
  uint16_t* sc = reinterpret_cast<uint16_t*>(scale_bf16_out);
  uint16_t* bi = reinterpret_cast<uint16_t*>(bias_bf16_out);
  if (group == 32)
    k_quantize<1><<<grid, 256, 0, s>>>(w, in_bf16, ngroups, cols / group, cols, bits, codes_out, sc, bi, ctrl);
  else if (group == 64)
    k_quantize<2><<<grid, 256, 0, s>>>(w, in_bf16, ngroups, cols / group, cols, bits, codes_out, sc, bi, ctrl);
  else
    k_quantize<4><<<grid, 256, 0, s>>>(w, in_bf16, ngroups, cols / group, cols, bits, codes_out, sc, bi, ctrl);
  return launch_status();
}

moe_status moe_pack_expert(const uint8_t* codes_gate, const void* scale_gate_bf16, const void* bias_gate_bf16,
                           const uint8_t* codes_up, const void* scale_up_bf16, const void* bias_up_bf16,
                           const uint8_t* codes_down, const void* scale_down_bf16, const void* bias_down_bf16,
                           int H, int I, int bits, int group, void* record_out, void* ws, void* stream) {
  const void* ptrs[10] = {codes_gate, scale_gate_bf16, bias_gate_bf16, codes_up, scale_up_bf16, bias_up_bf16,
                          codes_down, scale_down_bf16, bias_down_bf16, record_out};
  for (const void* q : ptrs) {
    if (!q) return MOE_ERR_INVALID_ARG;
    if (!aligned16(q)) return MOE_ERR_ALIGN;
  }
  if (ws && !aligned16(ws)) return MOE_ERR_ALIGN;
  if (moe_expert_bytes(H, I, bits, group) == 0) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  WsCtrl* ctrl = reinterpret_cast<WsCtrl*>(ws);
  const RecGeom g = rec_geom(H, I, bits, group);
  unsigned char* rec = reinterpret_cast<unsigned char*>(record_out);
  const unsigned maxg = (unsigned)num_sms() * 8;
  auto u16 = [](const void* q) { return reinterpret_cast<const uint16_t*>(q); };
  auto launch = [&](const TileSrc& src, int ntiles, int C, unsigned char* dst, uint32_t tile_bytes) {
    const int64_t ncode = (int64_t)ntiles * C / (bits == 3 ? 2 : 1);  // threads: (tile, group, lane, k-step[s])
    const int64_t nsb = (int64_t)ntiles * (C / group) * 8;
    const unsigned g1 = (unsigned)std::min<int64_t>((ncode + 255) / 256, maxg);
    const unsigned g2 = (unsigned)std::min<int64_t>((nsb + 255) / 256, maxg);
    if (bits == 4)
      k_pack_tile_codes<4><<<g1, 256, 0, s>>>(src, ntiles, C, group, dst, tile_bytes, g.blk, ctrl);
    else if (bits == 3)
      k_pack_tile_codes3<<<g1, 256, 0, s>>>(src, ntiles, C, group, dst, tile_bytes, g.blk, ctrl);
    else
      k_pack_tile_codes<2><<<g1, 256, 0, s>>>(src, ntiles, C, group, dst, tile_bytes, g.blk, ctrl);
    k_pack_tile_sb<<<g2, 256, 0, s>>>(src, ntiles, C, group, dst, tile_bytes, g.blk, g.blk - 64);
  };
  // gate/up tiles: gate rows then up rows of 8 units each
  launch(TileSrc{{codes_gate, codes_up}, {u16(scale_gate_bf16), u16(scale_up_bf16)},
                 {u16(bias_gate_bf16), u16(bias_up_bf16)}, 8},
         I / 8, H, rec, g.U);
  // down tiles: 16 rows each
  launch(TileSrc{{codes_down, codes_down}, {u16(scale_down_bf16), u16(scale_down_bf16)},
                 {u16(bias_down_bf16), u16(bias_down_bf16)}, 16},
         H / kTileRows, I, rec + g.down_off, g.D);
  return launch_status();
}

moe_status moe_router_topk(const void* x_bf16, const void* router_w_bf16, int B, int H, int E, int K, int renorm,
                           const int32_t* forced_idx, int32_t* idx_out, float* w_out, float* logits_out, void* ws,
                           size_t ws_bytes, void* stream) {
  if (!x_bf16 || !router_w_bf16 || !idx_out || !w_out) return MOE_ERR_INVALID_ARG;
  if (B <= 0 || B > MOEQ_MAX_B || H <= 0 || E <= 0 || K <= 0 || K > MOEQ_MAX_K || K > E) return MOE_ERR_INVALID_ARG;
  if (H % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (E > kRouterMaxE) return MOE_ERR_UNSUPPORTED;  // the selection holds 32 logits per lane
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_workspace_bytes(B, K, H, 32, E)) return MOE_ERR_WORKSPACE;
  if (!aligned16(x_bf16) || !aligned16(router_w_bf16) || !aligned16(ws)) return MOE_ERR_ALIGN;
  const size_t smem = std::max((size_t)std::min(B, kRouterTokTile) * H * 2, (size_t)std::min(B, kRouterTokTile) * E * 4);
  // a single token runs the one-token instance (one accumulator, a whole row's
  // loads in flight); batches tile eight tokens per CTA
  auto kern = B == 1 ? k_router_topk<1> : k_router_topk<kRouterTokTile>;
  if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_UNSUPPORTED;
  RouterParams p{};
  p.x = reinterpret_cast<const uint16_t*>(x_bf16);
  p.wr = reinterpret_cast<const uint16_t*>(router_w_bf16);
  p.forced = forced_idx;
  p.idx = idx_out;
  p.w = w_out;
  WsLayout wl = ws_layout(B, K, H, 32, E);
  p.logits = logits_out ? logits_out : reinterpret_cast<float*>((char*)ws + wl.logits);
  p.ctrl = reinterpret_cast<WsCtrl*>(ws);
  p.B = B;
  p.H = H;
  p.E = E;
  p.K = K;
  p.renorm = renorm;
  static_assert(MOEQ_MAX_B / kRouterTokTile <= (int)(sizeof(WsCtrl::router_ticket) / sizeof(unsigned)),
                "one router ticket per token tile");
  const int ctas = (E + kRouterWarps - 1) / kRouterWarps;
  const dim3 grid(ctas, (B + kRouterTokTile - 1) / kRouterTokTile);  // (B == 1: one tile either way)
  return launch_pdl(kern, grid, dim3(kRouterWarps * 32), smem, (cudaStream_t)stream, p);
}

moe_status moe_expert_ffn_q(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx, float* y_out,
                            void* ws, size_t ws_bytes, void* stream) {
  moe_status st = ffn_check_args(L, x_bf16, B, idx, y_out);
  if (st != MOE_OK) return st;
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_workspace_bytes(B, L->K, L->H, L->I, L->E)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_ALIGN;
  FfnParams p{};
  p.experts = reinterpret_cast<const uint8_t*>(L->experts);
  p.shared = reinterpret_cast<const uint8_t*>(L->shared);
  p.rec_r = moe_expert_bytes(L->H, L->I, L->bits_routed, L->group);
  p.geo_r = rec_geom(L->H, L->I, L->bits_routed, L->group);
  p.geo_s = rec_geom(L->H, L->I, L->bits_shared, L->group);
  p.x = reinterpret_cast<const uint16_t*>(x_bf16);
  p.idx = idx;
  WsLayout wl = ws_layout(B, L->K, L->H, L->I, L->E);
  p.h = reinterpret_cast<float*>((char*)ws + wl.h);
  p.y = y_out;
  p.ctrl = reinterpret_cast<WsCtrl*>(ws);
  p.H = L->H;
  p.I = L->I;
  p.E = L->E;
  p.K = L->K;
  p.G = L->group;
  p.bits_r = L->bits_routed;
  p.bits_s = L->bits_shared;
  p.B = B;
  cudaStream_t s = (cudaStream_t)stream;
  if (B > 1) {
    // a batch: group the picks by expert so that each active expert's tiles
    // are read once for all its tokens
    GrpParams gp{};
    gp.f = p;
    gp.g = GrpWs{reinterpret_cast<int*>((char*)ws + wl.cnt), reinterpret_cast<int*>((char*)ws + wl.off),
                 reinterpret_cast<int*>((char*)ws + wl.list), reinterpret_cast<int*>((char*)ws + wl.act),
                 reinterpret_cast<int*>((char*)ws + wl.nact)};
    const int max_act = std::min(p.E, B * p.K) + kGrpExtraChunks;  // routed work items at most
    const int ctas = kGrpCtasPerSm * num_sms();
    gp.nsh = (B + kGrpSharedTok - 1) / kGrpSharedTok;
    st = launch_pdl(k_group, dim3(1), dim3(256), (size_t)std::max(p.E + 1, B * p.K) * 4, s, idx, B, p.K, p.E, p.H, gp.g,
                    y_out,
                    p.ctrl);
    if (st != MOE_OK) return st;
    unsigned char* ximg = reinterpret_cast<unsigned char*>(ws) + wl.ximg;
    unsigned char* himg = reinterpret_cast<unsigned char*>(ws) + wl.himg;
    st = launch_pdl(k_stage_batch, dim3(B, 1), dim3(256), 0, s, x_bf16, 0, p.H, p.G, ximg, wl.ximg_stride,
                    wl.ximg_gs);
    if (st != MOE_OK) return st;
    gp.img = ximg;
    gp.img_stride = wl.ximg_stride;
    gp.img_gs_off = wl.ximg_gs;
    gp.tps = p.I / 8;
    gp.max_units = (gp.nsh + max_act) * gp.tps;
    const GrpKernels gk = grp_kernels(p.bits_r, p.bits_s, p.G);
    st = launch_pdl(gk.gate_up, dim3(ctas), dim3(kGrpWarps * 32), 0, s, gp);
    if (st != MOE_OK) return st;
    st = launch_pdl(k_stage_batch, dim3(B, p.K + 1), dim3(256), 0, s, (const void*)p.h, 1, p.I, p.G, himg,
                    wl.himg_stride, wl.himg_gs);
    if (st != MOE_OK) return st;
    gp.img = himg;
    gp.img_stride = wl.himg_stride;
    gp.img_gs_off = wl.himg_gs;
    gp.tps = p.H / kTileRows;
    gp.max_units = (gp.nsh + max_act) * gp.tps;
    return launch_pdl(gk.down, dim3(ctas), dim3(kGrpWarps * 32), 0, s, gp);
  }

  // one token: every CTA bulk-copies its share of whole tiles into shared memory
  p.dot_fma = batch1_dot_fma();
  size_t gu_bytes = 0, dn_bytes = 0;
  if (!ffn_plan(p, num_sms(), gu_bytes, dn_bytes)) return MOE_ERR_UNSUPPORTED;
  if (ensure_smem(k_gate_up, gu_bytes) != MOE_OK || ensure_smem(k_down, dn_bytes) != MOE_OK) return MOE_ERR_UNSUPPORTED;
  const int gu_tiles = (p.K + 1) * (p.I / 8), dn_jobs = (p.K + 1) * (p.H / kTileRows);
  p.dn_ctas = std::min(num_sms(), dn_jobs);
  st = launch_pdl(k_gate_up, dim3(std::min(num_sms(), gu_tiles)), dim3(kFfnWarps * 32), gu_bytes, s, p);
  if (st != MOE_OK) return st;
  return launch_pdl(k_down, dim3(p.dn_ctas), dim3(kFfnWarps * 32), dn_bytes, s, p);
}

moe_status moe_combine_residual(const moe_layer_q* L, const float* y, const float* w, const void* x_bf16,
                                const float* resid_in, int B, float* resid_out, void* xnorm_bf16_out, float eps,
                                void* stream) {
  if (!L || !y || !w || !x_bf16 || !resid_out) return MOE_ERR_INVALID_ARG;
  if (L->H <= 0 || L->K <= 0 || L->K > MOEQ_MAX_K || B <= 0 || B > MOEQ_MAX_B) return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(x_bf16) || !aligned16(resid_out) || (resid_in && !aligned16(resid_in)) ||
      (xnorm_bf16_out && !aligned16(xnorm_bf16_out)) || (L->shared_gate_w && !aligned16(L->shared_gate_w)))
    return MOE_ERR_ALIGN;
  CombineParams p{};
  p.y = y;
  p.w = w;
  p.x = reinterpret_cast<const uint16_t*>(x_bf16);
  p.resid_in = resid_in;
  p.gate_w = reinterpret_cast<const uint16_t*>(L->shared_gate_w);
  p.resid_out = resid_out;
  p.xnorm = reinterpret_cast<uint16_t*>(xnorm_bf16_out);
  p.B = B;
  p.H = L->H;
  p.K = L->K;
  p.eps = eps;
  return launch_pdl(k_combine, dim3(B * kCombineCluster), dim3(kCombineThreads), 0, (cudaStream_t)stream, p);
}

moe_status moe_get_device_error(void* ws, void* stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  int err = 0;
  if (cudaMemcpyAsync(&err, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  if (err != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
      (void)cudaGetLastError();
      return MOE_ERR_CUDA;
    }
  }
  return (moe_status)err;
}

}  // extern "C"

namespace moeq {
namespace {

// Shared-memory plans of the one-token gate/up and down kernels: the input
// image(s), the pieces' partial sums and as many tile buffers as the CTA's
// share needs (at most kFfnMaxBuf, and what fits). False when not one fits.
bool ffn_plan(FfnParams& p, int G, size_t& gu_bytes, size_t& dn_bytes) {
  const size_t budget = 227 * 1024 - 2 * 1024;  // leave room for the static shared memory
  auto cdiv = [](int a, int b) { return (a + b - 1) / b; };
  const int gu_total = (p.K + 1) * (p.I / 8), dn_total = (p.K + 1) * (p.H / kTileRows);
  // gate/up
  size_t o = align_up(qimg_plane_bytes(p.H), 128);
  p.gu_gs = (int)o;
  o += align_up(qimg_gs_bytes(p.H, p.G), 128);
  p.gu_xf = (int)o;
  if (p.dot_fma) o += align_up((size_t)p.H * 4, 128);
  const int gu_want = std::min(kFfnMaxBuf, cdiv(gu_total, std::min(G, gu_total)));
  p.gu_part = (int)o;
  o += align_up((size_t)gu_want * kFfnPiecesGu * kTileRows * 4, 128);
  p.gu_tiles = (int)o;
  p.gu_stride = (int)align_up(std::max(p.geo_r.U, p.geo_s.U), 128);
  if (o + (size_t)p.gu_stride > budget) return false;
  p.gu_nbuf = (int)std::min<size_t>(gu_want, (budget - o) / p.gu_stride);
  gu_bytes = o + (size_t)p.gu_nbuf * p.gu_stride;
  // down
  p.dn_img_gs = (int)align_up(qimg_plane_bytes(p.I), 128);
  p.dn_img_xf = p.dn_img_gs + (int)align_up(qimg_gs_bytes(p.I, p.G), 128);
  p.dn_img_stride = p.dn_img_xf + (p.dot_fma ? (int)align_up((size_t)p.I * 4, 128) : 0);
  o = (size_t)p.dn_img_stride * (p.K + 1);
  const int dn_want = std::min(kFfnMaxBuf, cdiv(dn_total, std::min(G, dn_total)));
  p.dn_part = (int)o;
  o += align_up((size_t)dn_want * kFfnPiecesDn * kTileRows * 4, 128);
  p.dn_tiles = (int)o;
  p.dn_stride = (int)align_up(std::max(p.geo_r.D, p.geo_s.D), 128);
  if (o + (size_t)p.dn_stride > budget) return false;
  p.dn_nbuf = (int)std::min<size_t>(dn_want, (budget - o) / p.dn_stride);
  dn_bytes = o + (size_t)p.dn_nbuf * p.dn_stride;
  return true;
}

// The fused kernel's instance for (routed bits, shared bits, group):
// shared experts at 4 bits or at the routed width. Null when there is none.
using StackKernel = void (*)(StackParams);
StackKernel stack_kernel(int br, int bs, int G) {
#define MOEQ_STACK_CASE(R, S, Gp, KS) \
  if (br == R && bs == S && G == Gp) return k_decode_layers<R, S, KS>;
#define MOEQ_STACK_GROUPS(R, S)  \
  MOEQ_STACK_CASE(R, S, 64, 2)   \
  MOEQ_STACK_CASE(R, S, 128, 4)
  MOEQ_STACK_GROUPS(4, 4)
  MOEQ_STACK_GROUPS(2, 4)
  MOEQ_STACK_GROUPS(3, 4)
  MOEQ_STACK_GROUPS(2, 2)
  MOEQ_STACK_GROUPS(3, 3)
  MOEQ_STACK_CASE(4, 4, 32, 1)
  MOEQ_STACK_CASE(2, 4, 32, 1)
  MOEQ_STACK_CASE(2, 2, 32, 1)
#undef MOEQ_STACK_GROUPS
#undef MOEQ_STACK_CASE
  return nullptr;
}

// Static shared memory of a fused-kernel instance (bytes).
size_t stack_static_smem(StackKernel kern) {
  cudaFuncAttributes fa{};
  size_t bytes = 0;
  if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess) bytes = fa.sharedSizeBytes;
  else (void)cudaGetLastError();
  return bytes ? bytes : 16 * 1024;  // unknown: leave a generous margin
}

// Shared-memory plan of the fused decode kernel; false when it does not fit.
bool stack_plan(StackParams& p, int G, size_t static_smem) {
  const int H = p.H, I = p.I, K = p.K;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o += align_up(bytes, 128);
    return (int)at;
  };
  auto cdiv = [](int a, int b) { return (a + b - 1) / b; };
  p.sm_xs = take((size_t)H * 2);
  p.sm_xplanes = take(qimg_plane_bytes(H));
  p.sm_xgs = take(qimg_gs_bytes(H, p.G));
  p.hplanes_stride = (int)align_up(qimg_plane_bytes(I), 128);
  p.hgs_stride = (int)align_up(qimg_gs_bytes(I, p.G), 128);
  p.sm_hplanes = take((size_t)p.hplanes_stride * (K + 1));
  p.sm_hgs = take((size_t)p.hgs_stride * (K + 1));
  const int ntiles_max = cdiv(I / 8, G) + cdiv(K * (I / 8), G) + 1;
  const int nd_max = cdiv(H / kTileRows, G);
  if (ntiles_max > kMaxTiles || nd_max > kMaxDnTiles) return false;
  p.sm_gpart = take(((size_t)cdiv(I / 8, G) * kGuPiecesShared + (size_t)(cdiv(K * (I / 8), G) + 1) * kGuPieces) *
                    kTileRows * 4);
  p.sm_dpart = take((size_t)nd_max * (K + 1) * kDnPieces * kTileRows * 4);
  // a ring slot holds two router rows, half of a gate/up tile or the CTA's
  // down tiles of one slot
  const int ng = H / p.G;
  const size_t half_tile = (size_t)std::max(quarter_lo(2, ng), ng - quarter_lo(2, ng)) *
                           std::max(p.geo_r.blk, p.geo_s.blk);
  const size_t down_item = (size_t)nd_max * std::max(p.geo_r.D, p.geo_s.D);
  p.slot_bytes = (int)align_up(std::max(std::max((size_t)2 * H * 2, half_tile), down_item), 128);
  const size_t budget = 227 * 1024 - align_up(static_smem, 1024);  // room for the static shared memory
  if (o + (size_t)p.slot_bytes * 2 > budget) return false;
  p.nslot = (int)std::min<size_t>(kMaxSlots, (budget - o) / p.slot_bytes);
  p.sm_ring = take((size_t)p.slot_bytes * p.nslot);
  return o <= budget;
}

size_t stack_smem_bytes(const StackParams& p) { return (size_t)p.sm_ring + (size_t)p.slot_bytes * p.nslot; }

}  // namespace
}  // namespace moeq

extern "C" moe_status moe_decode_layers(const moe_layer_q* layers, int n_layers, const void* x_bf16,
                                        const float* resid_in, int renorm, const int32_t* forced_idx,
                                        int32_t* idx_out, float* w_out, float* resid_out, void* xnorm_bf16_out,
                                        float eps, void* ws, size_t ws_bytes, void* stream) {
  if (!layers || n_layers <= 0 || n_layers > kStackMaxLayers) return MOE_ERR_INVALID_ARG;
  const moe_layer_q& L0 = layers[0];
  for (int l = 0; l < n_layers; ++l) {
    moe_status st = check_layer(&layers[l]);
    if (st != MOE_OK) return st;
    const moe_layer_q& L = layers[l];
    if (L.H != L0.H || L.I != L0.I || L.E != L0.E || L.K != L0.K || L.group != L0.group ||
        L.bits_routed != L0.bits_routed || L.bits_shared != L0.bits_shared)
      return MOE_ERR_INVALID_ARG;
  }
  if (!x_bf16 || !resid_out) return MOE_ERR_INVALID_ARG;
  if (!(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x_bf16) || !aligned16(resid_out) || (resid_in && !aligned16(resid_in)) ||
      (xnorm_bf16_out && !aligned16(xnorm_bf16_out)) || (ws && !aligned16(ws)))
    return MOE_ERR_ALIGN;
  if (!ws) return MOE_ERR_WORKSPACE;
  if (ws_bytes < moe_workspace_bytes(1, L0.K, L0.H, L0.I, L0.E)) return MOE_ERR_WORKSPACE;
  const int G = num_sms();
  auto cdiv = [](int a, int b) { return (a + b - 1) / b; };
  if (L0.E > kStackMaxE || cdiv(L0.E, G) > kMaxRouterRowsPerCta || G > kStackMaxCtas) return MOE_ERR_UNSUPPORTED;
  const int tps = L0.I / 8;
  if (cdiv(cdiv(L0.E, G), 2) + 2 * (cdiv(tps, G) + cdiv(L0.K * tps, G) + 1) + L0.K + 1 > kMaxItems)
    return MOE_ERR_UNSUPPORTED;
  if (L0.H % 32 != 0 || L0.H / 16 > kCThreads) return MOE_ERR_UNSUPPORTED;

  StackParams p{};
  for (int l = 0; l < n_layers; ++l) {
    p.L[l].experts = reinterpret_cast<const uint8_t*>(layers[l].experts);
    p.L[l].shared = reinterpret_cast<const uint8_t*>(layers[l].shared);
    p.L[l].router_w = reinterpret_cast<const uint16_t*>(layers[l].router_w);
    p.L[l].gate_w = reinterpret_cast<const uint16_t*>(layers[l].shared_gate_w);
  }
  p.n_layers = n_layers;
  p.H = L0.H;
  p.I = L0.I;
  p.E = L0.E;
  p.K = L0.K;
  p.G = L0.group;
  p.bits_r = L0.bits_routed;
  p.bits_s = L0.bits_shared;
  p.rec_r = moe_expert_bytes(p.H, p.I, p.bits_r, p.G);
  p.geo_r = rec_geom(p.H, p.I, p.bits_r, p.G);
  p.geo_s = rec_geom(p.H, p.I, p.bits_s, p.G);
  p.x_in = reinterpret_cast<const uint16_t*>(x_bf16);
  p.resid_in = resid_in;
  p.forced = forced_idx;
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.resid_out = resid_out;
  p.xnorm_out = reinterpret_cast<uint16_t*>(xnorm_bf16_out);
  p.eps = eps;
  p.renorm = renorm;
  WsLayout wl = ws_layout(1, p.K, p.H, p.I, p.E);
  p.ctrl = reinterpret_cast<WsCtrl*>(ws);
  p.logits = reinterpret_cast<float*>((char*)ws + wl.logits);
  p.h = reinterpret_cast<float*>((char*)ws + wl.h);
  p.r = reinterpret_cast<float*>((char*)ws + wl.r);
  p.sync = reinterpret_cast<WsCtrl*>(ws)->sync;
  p.ss_part = reinterpret_cast<float*>((char*)ws + wl.ss);
#ifdef MOEQ_STACK_TRACE
  // timeline builds: the phase stamps go right after the workspace proper
  const size_t trace_bytes = (size_t)n_layers * kTracePhases * G * sizeof(unsigned long long);
  p.trace = ws_bytes >= wl.total + trace_bytes ? reinterpret_cast<unsigned long long*>((char*)ws + wl.total) : nullptr;
#else
  p.trace = nullptr;
#endif
  const StackKernel kern = stack_kernel(p.bits_r, p.bits_s, p.G);
  if (!kern) return MOE_ERR_UNSUPPORTED;
  static std::mutex mu;
  static size_t static_smem[64] = {};  // per instance, read once (the instances' addresses are fixed)
  static StackKernel seen[64] = {};
  size_t ss = 0;
  std::unique_lock<std::mutex> lock(mu);
  for (int i = 0; i < 64 && !ss; ++i) {
    if (seen[i] == kern) ss = static_smem[i];
    else if (!seen[i]) {
      seen[i] = kern;
      ss = static_smem[i] = stack_static_smem(kern);
    }
  }
  lock.unlock();
  if (!stack_plan(p, G, ss ? ss : 16 * 1024)) return MOE_ERR_UNSUPPORTED;
  const size_t smem = stack_smem_bytes(p);
  if (ensure_smem(kern, smem) != MOE_OK) return MOE_ERR_UNSUPPORTED;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kStackThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs co-resident: they wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
