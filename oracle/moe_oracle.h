/*
 * moe_oracle.h -- the oracle: a plain, slow, single-threaded C99 restatement
 * in fp64 of the decode-time quantized MoE FFN step.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the benchmark's
 * CPU-baseline leg may load it; the library's own code path never does. It
 * shares no code, header, table or helper with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *  [FM]   "Flash-MoE - Chay mo hinh 397 ty tham so tren laptop"
 *         (vi.news.hada.io/topic?id=27758):
 *           - section "Kien truc mo hinh": 512 experts per layer, K=4 active
 *             per token, hidden size 4096;
 *           - section "SSD Expert Streaming": one expert is about 6.75 MB;
 *           - section "Kernel dequant toi uu FMA": (nibble*scale+bias)*x
 *             rewritten as fma(nibble, scale*x, bias*x);
 *           - section "Metal Compute Shaders": 4-bit/2-bit dequant mat-vec,
 *             SwiGLU, RMS norm, MoE combine + residual + gate;
 *           - section "Deferred GPU Expert Compute": combine + norm + residual
 *             run on the GPU and feed the next layer.
 *  [LOOM] "LOOM" (alessandroviola.dev/it/research/loom/): expert-major
 *         storage (each expert's data kept contiguous).
 *
 * Readings taken where the pages are silent:
 *  - q is unsigned (0..2^b-1), b in {2, 3, 4}; w = q*scale + bias per group
 *    of G consecutive input elements; scale and bias are bf16.
 *  - quantisation (weights -> codes) is min-max per group: bias = the
 *    group's minimum, scale = its range / (2^b - 1), codes rounded to
 *    nearest; 3 bits as the Autoresearch page's size/quality point
 *    ("Autoresearch impulsa ... 20.34 tok/s", "Optimizaciones Efectivas").
 *  - packing is row-major, low bits first; the (scale, bias) pair of each
 *    (row, group) is stored interleaved, scale first.
 *  - an expert record is gate [I,H], up [I,H], down [H,I] packed codes, then
 *    the gate, up and down (scale, bias) tables.
 *  - router: logits = W_r x; softmax over all E; the K largest logits in
 *    descending order, ties to the lower index; w_k = p[idx_k], optionally
 *    renormalised over the K picks.
 *  - SwiGLU: h = silu(g) * u with silu(z) = z / (1 + exp(-z)).
 *  - combine: out = r + sum_k w_k y_k + gamma * y_shared, gamma = 1, or
 *    sigmoid(w_sg . x) when a shared-gate vector is given.
 *  - norm between stacked layers: RMSNorm with unit weight, then bf16 (RNE).
 *
 * Pins (tests/test_oracle_pins.py): golden pack bytes, the 6.75 MB expert
 * size, the three equal forms of the dequant dot product, constant-code and
 * zero-code closed forms, one-hot inputs, brute-force top-K, textbook SwiGLU
 * values, closed-form softmax and RMSNorm cases, and combine special cases.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bf16 <-> fp64 (exact widening; RNE narrowing from fp64) */
double moe_ref_bf16_to_f64(uint16_t b);
uint16_t moe_ref_f64_to_bf16(double v);

/* bytes of one packed expert record (gate, up, down codes + their tables) */
size_t moe_ref_expert_bytes(int H, int I, int bits, int group);

/* packing of one [rows, cols] code matrix at bits in {2, 3, 4}; returns 0,
 * or 1 on bad arguments or a code that does not fit in `bits` bits */
int moe_ref_pack(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                 int rows, int cols, int bits, int group, uint8_t* packed, uint16_t* sb);
int moe_ref_unpack(const uint8_t* packed, const uint16_t* sb, int rows, int cols, int bits,
                   int group, uint8_t* codes, uint16_t* scale, uint16_t* bias);

/* min-max group-affine quantisation of fp32 weights [rows, cols] into codes
 * u8 [rows, cols] and bf16 scale/bias [rows, cols/group]; the codes are
 * decided in binary32 like the GPU kernel (see moe_oracle.c); 0, or 1 on bad
 * arguments or a non-finite weight */
int moe_ref_quantize(const float* w, int rows, int cols, int bits, int group,
                     uint8_t* codes, uint16_t* scale, uint16_t* bias);

/* y[r] = sum_c (q[r,c]*s[r,g(c)] + b[r,g(c)]) * x[c], three written-out forms */
void moe_ref_dequant_gemv(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                          int rows, int cols, int group, const double* x, double* y);
void moe_ref_dequant_gemv_fma(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                              int rows, int cols, int group, const double* x, double* y);
void moe_ref_dequant_gemv_grouped(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                                  int rows, int cols, int group, const double* x, double* y);

/* router: logits[e] = sum_h W_r[e,h] x[h]  (one token) */
void moe_ref_router_logits(const uint16_t* x_bf16, const uint16_t* wr_bf16, int H, int E, double* logits);
void moe_ref_softmax(const double* logits, int E, double* p);
/* top-K (forced == NULL) or forced indices; returns 0, 1 on bad arguments */
int moe_ref_topk(const double* logits, int E, int K, int renorm, const int32_t* forced,
                 int32_t* idx, double* w);

double moe_ref_silu(double z);
void moe_ref_swiglu(const double* g, const double* u, int n, double* h);

/* one expert: y = W_d (silu(W_g x) * (W_u x)); x has H entries, y has H */
void moe_ref_expert_ffn(int H, int I, int group,
                        const uint8_t* codes_g, const uint16_t* scale_g, const uint16_t* bias_g,
                        const uint8_t* codes_u, const uint16_t* scale_u, const uint16_t* bias_u,
                        const uint8_t* codes_d, const uint16_t* scale_d, const uint16_t* bias_d,
                        const double* x, double* y);

double moe_ref_shared_gate(const uint16_t* wsg_bf16, const uint16_t* x_bf16, int H);

/* out = r + sum_{k<K} w[k] y[k] + gamma * y[K]; y is [K+1, H] */
void moe_ref_combine(int H, int K, const double* y, const double* w, double gamma,
                     const double* r, double* out);

void moe_ref_rmsnorm(const double* v, int H, double eps, double* out);
void moe_ref_rmsnorm_bf16(const double* v, int H, double eps, uint16_t* out);
/* out[i] = bf16(v[i] / sqrt(mean(v^2) + eps) * w[i]); w == NULL: unit weight */
void moe_ref_rmsnorm_weighted_bf16(const double* v, const uint16_t* w, int H, double eps, uint16_t* out);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ORACLE_H */
