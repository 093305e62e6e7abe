/*
 * moeq.h -- C ABI of libmoeq.so: the decode-time quantized Mixture-of-Experts
 * FFN step on NVIDIA B200 (sm_100a).
 *
 * One token (or a small batch of tokens) passes through one MoE layer:
 *   1. router GEMV, logits = W_r x, then softmax and top-K over E experts;
 *   2. for each selected expert and for the always-on shared expert, the
 *      gate and up projections as group-affine low-bit dequant mat-vecs,
 *      w = q*scale + bias per group of G consecutive inputs, evaluated in the
 *      rearranged form fma(q, scale*x, bias*x) summed per group;
 *   3. SwiGLU, h = silu(gate) * up;
 *   4. the down projection, a dequant mat-vec of h;
 *   5. the weighted combine with the shared expert and the residual, with an
 *      optional RMSNorm'd bf16 copy for the next layer.
 *
 * Sources, cited by page title and section:
 *   "Flash-MoE - Chay mo hinh 397 ty tham so tren laptop"
 *   (vi.news.hada.io/topic?id=27758):
 *     "Kien truc mo hinh"           512 experts, K=4 active, hidden 4096;
 *     "SSD Expert Streaming"        about 6.75 MB per 4-bit expert;
 *     "Kernel dequant toi uu FMA"   (nibble*scale+bias)*x as
 *                                   fma(nibble, scale*x, bias*x);
 *     "Metal Compute Shaders"       4-bit/2-bit dequant mat-vec, SwiGLU,
 *                                   RMS norm, MoE combine + residual + gate;
 *     "Deferred GPU Expert Compute" combine + norm + residual on the GPU,
 *                                   handed straight to the next layer.
 *   "LOOM" (alessandroviola.dev/it/research/loom/): expert-major storage.
 *
 * Conventions for every call:
 *   - Pointers named *_bf16 hold IEEE bfloat16 values; all buffers except the
 *     moe_layer_q struct itself are DEVICE memory owned by the caller. The
 *     library never allocates or frees device memory.
 *   - Device pointers must be 16-byte aligned (MOE_ERR_ALIGN otherwise).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise, except moe_get_device_error.
 *   - Argument errors are found on the host before any launch and returned
 *     as a status; nothing is launched then.
 *   - Errors found on the device (an expert index outside [0, E), a code
 *     that does not fit its bit width) set an error word in the workspace
 *     and the affected output is written as zero; kernels never trap.
 *     Read it with moe_get_device_error.
 *   - A workspace is caller-allocated device memory of at least
 *     moe_workspace_bytes(...) bytes, zeroed once with moe_workspace_init
 *     before first use. Calls that share a workspace must be ordered on one
 *     stream; distinct workspaces make calls independent.
 */
#ifndef MOEQ_H
#define MOEQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOEQ_ABI_VERSION 1
#define MOEQ_MAX_K 8      /* largest routed top-K */
#define MOEQ_MAX_B 128    /* largest token batch per call */
#define MOEQ_STATIC_SCRATCH_BYTES (2u << 20) /* scratch of moe_expert_ffn_q_static, per GPU */

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size or shape */
  MOE_ERR_ALIGN = 2,       /* a device pointer is not 16-byte aligned */
  MOE_ERR_UNSUPPORTED = 3, /* bits/group/shape outside the supported set */
  MOE_ERR_CUDA = 4,        /* a CUDA launch or copy failed */
  MOE_ERR_INDEX = 5,       /* device: an expert index was outside [0, E) */
  MOE_ERR_TIMEOUT = 6,     /* device: a bounded wait gave up */
  MOE_ERR_WORKSPACE = 7,   /* workspace missing or smaller than required */
  MOE_ERR_RANGE = 8        /* device: a code did not fit in its bit width */
} moe_status;

/*
 * One MoE layer's resident weights (all pointers are device memory).
 *
 * Expert record (expert-major: each expert is one contiguous block, as in
 * LOOM's layout), for `bits` in {2, 3, 4} and group size `group`; the
 * dequantised weight is w = q*scale + bias with q unsigned and one bf16
 * (scale, bias) pair per row and group of `group` inputs. Every matrix is
 * stored as tiles of 16 rows laid out for the int8 tensor-core dot: a tile
 * holds, for each group g, one block of
 *   codes: 32 lanes x (group/32 k-steps) x W bytes (W = 8 at 4 bits, 4 at
 *          2 bits); lane 4*r + t of k-step j holds the codes of inputs
 *          g*group + 32j + 8t .. +7 of local rows r and r+8: at 4 bits two
 *          words, input 8t+i at nibble i; at 2 bits one word, input 8t+2i of
 *          row r at bits 8i, of row r+8 at 8i+2, input 8t+2i+1 of row r at
 *          8i+4, of row r+8 at 8i+6. At 3 bits (group 64 or 128) the low two
 *          bits of every code form such a 2-bit plane (4 bytes per lane and
 *          k-step), followed by a plane of the third bits (2 bytes per lane
 *          and k-step, lane L at byte 128*(group/32) + 2*L*(group/32)): in
 *          the word of k-steps 2p and 2p+1, bit 8i + 4*(j & 1) + s holds the
 *          third bit of the code at bit 8i + 2s of k-step j's 2-bit word
 *   tables: 8 x [(scale, bias) of local row r][(scale, bias) of row r+8]
 * The record is I/8 gate/up tiles of H inputs (tile T: gate rows 8T..8T+7
 * as local rows 0..7, up rows 8T..8T+7 as 8..15), then H/16 down tiles of I
 * inputs (tile T: rows 16T..16T+15). moe_expert_layout gives the sizes;
 * moe_pack_expert writes a record. At H=4096, I=1024, 4-bit, group 64 a
 * record is 7,077,888 bytes (6.75 MiB), the per-expert size the Flash-MoE
 * page gives ("SSD Expert Streaming").
 */
typedef struct moe_layer_q {
  int H;           /* hidden size; H*bits/8 and I*bits/8 multiples of 16 */
  int I;           /* expert intermediate size */
  int E;           /* routed experts */
  int K;           /* routed experts per token, 1..MOEQ_MAX_K, K <= E */
  int group;       /* 32, 64 or 128; divides H and I */
  int bits_routed; /* 2, 3 or 4 (3: group 64 or 128) */
  int bits_shared; /* 2, 3 or 4 */
  const void* experts;       /* E routed records, back to back */
  const void* shared;        /* 1 shared-expert record (bits_shared) */
  const void* router_w;      /* bf16 [E, H], row-major */
  const void* shared_gate_w; /* bf16 [H], or NULL: shared expert weight 1 */
} moe_layer_q;

/* Bytes of one expert record (see moe_layer_q); 0 for unsupported args. */
size_t moe_expert_bytes(int H, int I, int bits, int group);

/* Layout of one expert record (see moe_layer_q):
 *   lay[0] bytes of one gate/up tile ((H/group) blocks)
 *   lay[1] byte offset of the first down tile (= lay[5] * lay[0])
 *   lay[2] bytes of one down tile ((I/group) blocks)
 *   lay[3] rows per tile (16)
 *   lay[4] bytes of one block (codes, then 64 bytes of tables)
 *   lay[5] gate/up tiles (I/8) */
moe_status moe_expert_layout(int H, int I, int bits, int group, size_t lay[6]);

/* Workspace bytes for calls on up to B tokens of this layer shape. */
size_t moe_workspace_bytes(int B, int K, int H, int I, int E);

/* Zero a workspace (asynchronous cudaMemsetAsync on `stream`). */
moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/*
 * moe_workspace_debug -- testing hook for the bounded waits (the pages have
 * no counterpart). Sets two words of the workspace control block, in stream
 * order, for the calls that use the workspace afterwards:
 *   wait_budget_us  every bounded wait gives up after about this many
 *                   microseconds (0: the default, about one second)
 *   withhold_cta    c + 1: CTA c of moe_decode_layers skips its arrival on
 *                   the first layer's logits exchange, so every CTA's wait on
 *                   it runs out: the kernel then sets MOE_ERR_TIMEOUT, lets
 *                   its bulk copies land and exits; 0: off
 * moe_workspace_init clears both. MOE_ERR_WORKSPACE for a missing or short
 * workspace, MOE_ERR_ALIGN, MOE_ERR_INVALID_ARG for withhold_cta < 0.
 */
moe_status moe_workspace_debug(void* ws, size_t ws_bytes, unsigned wait_budget_us, int withhold_cta, void* stream);

/*
 * moe_pack_q -- pack one code matrix into the plain row-major interchange
 * image: code j of a row at bit offset (j*bits) mod 8 of byte j*bits/8 of
 * the row (low bits first), and the (scale, bias) bf16 pair of each (row,
 * group) interleaved, scale first. This image is for storage and exchange;
 * the resident expert record that moe_expert_ffn_q and moe_decode_layers
 * read is tile-major and is written by moe_pack_expert.
 *   codes      u8 [rows, cols], one code per byte, values < 2^bits
 *   scale_bf16 bf16 [rows, cols/group]
 *   bias_bf16  bf16 [rows, cols/group]
 *   packed_out u8 [rows, cols*bits/8]
 *   sb_out     bf16 [rows, cols/group, 2]  (scale, bias) pairs
 *   ws         optional workspace (NULL allowed): a code >= 2^bits sets
 *              MOE_ERR_RANGE there; its low `bits` bits are packed.
 * bits in {2,3,4} (a 3-bit code may straddle two bytes); group in
 * {32,64,128}; cols % group == 0; cols*bits/8 a multiple of 16 (at 3 bits:
 * cols % 128 == 0). The layout is the affine form of the Flash-MoE page
 * ("Kernel dequant toi uu FMA": (nibble*scale+bias)), 4- and 2-bit widths as
 * in its "Metal Compute Shaders" section, 3 bits as on the Autoresearch page
 * ("Optimizaciones Efectivas").
 */
moe_status moe_pack_q(const uint8_t* codes, const void* scale_bf16, const void* bias_bf16,
                      int rows, int cols, int bits, int group,
                      void* packed_out, void* sb_out, void* ws, void* stream);

/*
 * moe_quantize -- min-max group-affine quantisation of a weight matrix into
 * the codes and (scale, bias) that moe_pack_q and moe_pack_expert take: the
 * affine form w ~ q*scale + bias of the Flash-MoE page ("Kernel dequant toi
 * uu FMA"), at 2, 3 or 4 bits (3 bits: the size/quality point of the
 * Autoresearch page, "Optimizaciones Efectivas").
 *   w          weights [rows, cols]: fp32 (in_bf16 = 0) or bf16 (in_bf16 = 1)
 *   codes_out  u8 [rows, cols], one code per byte
 *   scale_bf16_out, bias_bf16_out  bf16 [rows, cols/group]
 *   ws         optional workspace (NULL allowed): a non-finite weight sets
 *              MOE_ERR_RANGE there and its group is written as zeros
 * Per (row, group of `group` inputs): lo, hi = the group's extreme weights;
 * scale = bf16((hi - lo) / (2^bits - 1)), bias = bf16(lo) (nearest even);
 * q = clamp(rint((w - bias) / scale), 0, 2^bits - 1), or 0 when the bf16
 * scale is 0. Each step is one binary32 operation rounded to nearest even,
 * so the codes are reproducible bit for bit. bits in {2,3,4}; group in
 * {32,64,128} dividing cols (the record of 3-bit experts needs group 64 or
 * 128). MOE_ERR_UNSUPPORTED / MOE_ERR_INVALID_ARG / MOE_ERR_ALIGN otherwise.
 */
moe_status moe_quantize(const void* w, int in_bf16, int rows, int cols, int bits, int group, uint8_t* codes_out,
                        void* scale_bf16_out, void* bias_bf16_out, void* ws, void* stream);

/*
 * moe_pack_expert -- pack the gate [I,H], up [I,H] and down [H,I] code
 * matrices of one expert (u8 codes, bf16 scale/bias [rows, cols/group]) into
 * one resident expert record at record_out (moe_expert_bytes(H, I, bits,
 * group) bytes) in the tile-major layout described at moe_layer_q. The
 * record holds the same codes and (scale, bias) pairs as the row-major image
 * of moe_pack_q, in a different order. ws as in moe_pack_q.
 */
moe_status moe_pack_expert(const uint8_t* codes_gate, const void* scale_gate_bf16, const void* bias_gate_bf16,
                           const uint8_t* codes_up, const void* scale_up_bf16, const void* bias_up_bf16,
                           const uint8_t* codes_down, const void* scale_down_bf16, const void* bias_down_bf16,
                           int H, int I, int bits, int group, void* record_out, void* ws, void* stream);

/*
 * moe_router_topk -- router GEMV + softmax + top-K for B tokens.
 *   x_bf16        bf16 [B, H]
 *   router_w_bf16 bf16 [E, H]
 *   forced_idx    NULL, or int32 [B, K]: use these experts instead of the
 *                 top-K (their weights still come from the softmax)
 *   idx_out       int32 [B, K]: experts by descending logit, ties to the
 *                 lower index
 *   w_out         fp32 [B, K]: softmax probability over all E of each pick;
 *                 divided by their sum when renorm != 0
 *   logits_out    fp32 [B, E] or NULL
 * Logits accumulate in fp32 (bf16 products are exact in fp32). NaN logits
 * rank as -inf; a pick left with no finite logit is -1 and sets
 * MOE_ERR_INDEX (its weight is 0). E <= 1024 (MOE_ERR_UNSUPPORTED above:
 * the selection holds 32 logits per lane of a warp).
 * Source: "Kien truc mo hinh" (512 experts, K active per token).
 */
moe_status moe_router_topk(const void* x_bf16, const void* router_w_bf16, int B, int H, int E, int K,
                           int renorm, const int32_t* forced_idx, int32_t* idx_out, float* w_out,
                           float* logits_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_expert_ffn_q -- gate/up dequant mat-vecs, SwiGLU and down dequant
 * mat-vec for the K routed experts idx[b, :] and the shared expert of each
 * token, in one call.
 *   x_bf16 bf16 [B, H]; idx int32 [B, K]
 *   y_out  fp32 [B, K+1, H]: slot k < K is expert idx[b,k]'s output, slot K
 *          the shared expert's (unweighted)
 * Per group of G inputs a row contributes scale*sum(q*x) + bias*sum(x): the
 * group-summed form of fma(q, scale*x, bias*x) (Flash-MoE page, section
 * "Kernel dequant toi uu FMA"). The inputs (x, then h) are rounded once to
 * 16-bit fixed point per group; code x input products and their group sums
 * are exact integers (tensor cores); scale, bias and the sum over groups are
 * fp32. Accuracy: each input moves by at most 2^-16 of its group's largest
 * magnitude, so a row's error is about 2^-16 * max|x| * ||w_row||_2 plus fp32
 * rounding, far inside the parity bar max|err| <= 2e-3 * ||y||_inf that the
 * tests hold every output to. An index outside [0,E) sets MOE_ERR_INDEX and
 * zeroes that slot. B up to MOEQ_MAX_B: batches (B > 1) are grouped per
 * expert so that each active expert's tiles cross HBM once per call.
 */
moe_status moe_expert_ffn_q(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx,
                            float* y_out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_combine_residual -- out[b] = r[b] + sum_k w[b,k] y[b,k] + gamma_b y[b,K]
 *   y fp32 [B, K+1, H]; w fp32 [B, K]; x_bf16 bf16 [B, H]
 *   resid_in   fp32 [B, H], or NULL: r = x (bf16 widened)
 *   gamma_b    1 when L->shared_gate_w is NULL, else sigmoid(w_sg . x[b])
 *   resid_out  fp32 [B, H] (may alias resid_in)
 *   xnorm_bf16_out  bf16 [B, H] or NULL: RMSNorm(out[b]) with unit weight
 *              and epsilon eps, rounded to nearest-even bf16 (each token's
 *              sum of squares is gathered across a cluster of 8 CTAs; a part
 *              that has not arrived after about a second leaves that CTA's
 *              eighth of the row NaN instead of waiting on)
 * Source: "Metal Compute Shaders" (MoE combine + residual + gate, RMS norm)
 * and "Deferred GPU Expert Compute" (combine + norm + residual feed the next
 * layer).
 */
moe_status moe_combine_residual(const moe_layer_q* L, const float* y, const float* w, const void* x_bf16,
                                const float* resid_in, int B, float* resid_out, void* xnorm_bf16_out,
                                float eps, void* stream);

/*
 * moe_decode_layers -- one token (batch 1) through n_layers MoE layers of the
 * same shape in ONE persistent launch: for each layer l the router, softmax
 * and top-K, the gate/up dequant mat-vecs with SwiGLU, the down dequant
 * mat-vec, the combine with the shared expert and the residual, then the
 * next layer's input x_{l+1} = bf16(RMSNorm(r_{l+1})), as the Flash-MoE page
 * chains them ("Deferred GPU Expert Compute": combine + norm + residual stay
 * on the GPU and feed the next layer). Results equal chaining
 * moe_router_topk, moe_expert_ffn_q and moe_combine_residual per layer.
 *   layers      host array of n_layers (1..64) layer descriptors
 *   x_bf16      bf16 [H]: input of layer 0
 *   resid_in    fp32 [H] residual of layer 0, or NULL: r_0 = x (widened)
 *   forced_idx  int32 [n_layers, K] or NULL (as in moe_router_topk)
 *   idx_out, w_out  int32 / fp32 [n_layers, K] or NULL: picks and weights
 *   resid_out   fp32 [H]: r_n
 *   xnorm_bf16_out  bf16 [H] or NULL: bf16(RMSNorm(r_n))
 * Needs one CTA per SM for the whole launch (co-resident; cooperative
 * launch), E <= 1024, H/16 <= 512, a shared-memory plan that fits one SM,
 * and a shared expert at 4 bits or at the routed width (MOE_ERR_UNSUPPORTED
 * otherwise; use the per-call path). A wait that
 * exceeds about one second ends the kernel with MOE_ERR_TIMEOUT in the
 * workspace, which must then be re-initialised with moe_workspace_init.
 */
moe_status moe_decode_layers(const moe_layer_q* layers, int n_layers, const void* x_bf16, const float* resid_in,
                             int renorm, const int32_t* forced_idx, int32_t* idx_out, float* w_out,
                             float* resid_out, void* xnorm_bf16_out, float eps, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * moe_rmsnorm -- x[b] = bf16(r[b] / sqrt(mean(r[b]^2) + eps) * weight), the
 * RMS norm of the Flash-MoE page ("Metal Compute Shaders": a kernel of its
 * own between the MoE block and the next layer), rounded to nearest-even
 * bf16.
 *   r            fp32 [B, H]
 *   weight_bf16  bf16 [H], or NULL for unit weight
 *   xnorm_bf16_out  bf16 [B, H]
 * H a multiple of 8 (MOE_ERR_UNSUPPORTED otherwise); eps >= 0. The same
 * norm is fused into moe_combine_residual and moe_decode_layers (unit
 * weight there).
 */
moe_status moe_rmsnorm(const float* r, const void* weight_bf16, int B, int H, float eps, void* xnorm_bf16_out,
                       void* stream);

/* Read (and clear) the workspace error word. Synchronises `stream`.
 * Returns MOE_OK, MOE_ERR_INDEX, MOE_ERR_RANGE, MOE_ERR_TIMEOUT, or
 * MOE_ERR_CUDA if the copy itself failed. */
moe_status moe_get_device_error(void* ws, void* stream);

/*
 * moe_expert_ffn_q_static -- moe_expert_ffn_q without a caller workspace,
 * for callers that cannot allocate device memory: code handed only its
 * input and output buffers by a runtime that owns all device allocation, or
 * code running where cudaMalloc may not be called. (The pages describe no
 * such call; it is a convenience of this library.)
 *   L, x_bf16, B, idx, y_out, stream  as in moe_expert_ffn_q
 *   error_out  int32 device word, or NULL: receives the call's device error
 *              in stream order: 0, MOE_ERR_INDEX when an index was outside
 *              [0,E) and its slot was zeroed, or MOE_ERR_TIMEOUT when a
 *              bounded wait for a tile copy ran out (about one second)
 * Scratch is a MOEQ_STATIC_SCRATCH_BYTES array inside the library, held by
 * every GPU that loads it until the process exits. A shape whose
 * moe_workspace_bytes(B, K, H, I, E) exceeds that size is rejected with
 * MOE_ERR_WORKSPACE; every argument error (those of moe_expert_ffn_q first)
 * returns before anything is queued. The call allocates nothing:
 * it clears the array's control block with cudaMemsetAsync and runs the
 * kernels of moe_expert_ffn_q on the array. All calls on a device share the
 * array and it keeps the last call's contents, so calls that overlap on the
 * GPU (different streams or host threads) race and must be ordered by the
 * caller. The first call on each device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.
 */
moe_status moe_expert_ffn_q_static(const moe_layer_q* L, const void* x_bf16, int B, const int32_t* idx,
                                   float* y_out, int32_t* error_out, void* stream);

const char* moe_status_str(moe_status s);
int moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOEQ_H */
