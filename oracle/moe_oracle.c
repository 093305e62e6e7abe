/*
 * moe_oracle.c -- the oracle (test infrastructure only; see moe_oracle.h for
 * the sources, the readings taken and the rule on who may call it).
 *
 * Everything is fp64 with naive loops, in the order the method states it.
 * Build: gcc -std=c99 -O2 -ffp-contract=off.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- bf16 <-> fp64 ------------------------------------------------------ */

/* A bf16 value is the upper half of an IEEE binary32; widening is exact. */
double moe_ref_bf16_to_f64(uint16_t b) {
  union { uint32_t u; float f; } v;
  v.u = (uint32_t)b << 16;
  return (double)v.f;
}

/* Nearest bf16 to v, ties to even significand (finite v only; overflow
 * saturates to infinity). bf16 keeps 8 significant bits, exponent range as
 * binary32, subnormal quantum 2^-133. */
uint16_t moe_ref_f64_to_bf16(double v) {
  double a = fabs(v);
  uint16_t sign = signbit(v) ? 0x8000u : 0u;
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e); /* a = m * 2^e, 0.5 <= m < 1 */
  double quantum = (e - 1 >= -126) ? ldexp(1.0, e - 8) : ldexp(1.0, -133);
  double k = nearbyint(a / quantum); /* default rounding: nearest, ties to even */
  double r = k * quantum;
  if (r > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80u); /* > max bf16 */
  union { uint32_t u; float f; } f;
  f.f = (float)r; /* exact: r is a bf16 value */
  return (uint16_t)(sign | (uint16_t)(f.u >> 16));
}

/* ---- sizes and packing ------------------------------------------------- */

/* Expert record = gate [I,H] + up [I,H] + down [H,I]: 3*H*I codes of `bits`
 * bits, plus one (scale, bias) bf16 pair (4 bytes) per group of `group`
 * inputs in each row. At H=4096, I=1024, 4-bit, group 64 this is
 * 6,291,456 + 786,432 = 7,077,888 bytes = 6.75 MiB: the per-expert size the
 * Flash-MoE page gives (section "SSD Expert Streaming"). */
size_t moe_ref_expert_bytes(int H, int I, int bits, int group) {
  size_t weights = 3u * (size_t)H * (size_t)I;
  return weights * (size_t)bits / 8u + weights / (size_t)group * 4u;
}

static int pack_args_ok(int rows, int cols, int bits, int group) {
  if (rows < 0 || cols <= 0) return 0;
  if (bits < 2 || bits > 4) return 0;
  if (group <= 0 || cols % group != 0) return 0;
  if ((cols * bits) % 8 != 0) return 0;
  return 1;
}

/* Code q[r,c] occupies bits c*bits .. c*bits + bits - 1 of row r's packed
 * bytes, read as one little-endian bit string (bit k is bit k%8 of byte
 * k/8), lowest code bit first; at 3 bits a code may straddle two bytes. The
 * (scale, bias) of group g of row r is the bf16 pair sb[2*(r*ng+g)],
 * sb[2*(r*ng+g)+1]. */
int moe_ref_pack(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                 int rows, int cols, int bits, int group, uint8_t* packed, uint16_t* sb) {
  if (!codes || !scale || !bias || !packed || !sb) return 1;
  if (!pack_args_ok(rows, cols, bits, group)) return 1;
  size_t row_bytes = (size_t)cols * bits / 8;
  int ng = cols / group;
  memset(packed, 0, row_bytes * (size_t)rows);
  for (int r = 0; r < rows; ++r) {
    uint8_t* row = packed + (size_t)r * row_bytes;
    for (int c = 0; c < cols; ++c) {
      unsigned q = codes[(size_t)r * cols + c];
      if (q >> bits) return 1;
      for (int i = 0; i < bits; ++i) {
        size_t k = (size_t)c * bits + i;
        if ((q >> i) & 1u) row[k / 8] |= (uint8_t)(1u << (k % 8));
      }
    }
    for (int g = 0; g < ng; ++g) {
      size_t rg = (size_t)r * ng + g;
      sb[2 * rg] = scale[rg];
      sb[2 * rg + 1] = bias[rg];
    }
  }
  return 0;
}

int moe_ref_unpack(const uint8_t* packed, const uint16_t* sb, int rows, int cols, int bits,
                   int group, uint8_t* codes, uint16_t* scale, uint16_t* bias) {
  if (!codes || !scale || !bias || !packed || !sb) return 1;
  if (!pack_args_ok(rows, cols, bits, group)) return 1;
  size_t row_bytes = (size_t)cols * bits / 8;
  int ng = cols / group;
  for (int r = 0; r < rows; ++r) {
    const uint8_t* row = packed + (size_t)r * row_bytes;
    for (int c = 0; c < cols; ++c) {
      unsigned q = 0;
      for (int i = 0; i < bits; ++i) {
        size_t k = (size_t)c * bits + i;
        q |= (unsigned)((row[k / 8] >> (k % 8)) & 1u) << i;
      }
      codes[(size_t)r * cols + c] = (uint8_t)q;
    }
    for (int g = 0; g < ng; ++g) {
      size_t rg = (size_t)r * ng + g;
      scale[rg] = sb[2 * rg];
      bias[rg] = sb[2 * rg + 1];
    }
  }
  return 0;
}

/* ---- quantisation ------------------------------------------------------ */

/* Min-max group-affine quantisation of fp32 weights into the pages' affine
 * form w ~ q*scale + bias (Flash-MoE page, "Kernel dequant toi uu FMA"), at
 * 2, 3 or 4 bits (3 bits: the size/quality point of the Autoresearch page,
 * "Optimizaciones Efectivas"). Per (row, group of `group` inputs):
 *   lo, hi = min and max of the group's weights;
 *   scale  = bf16((hi - lo) / (2^bits - 1)),  bias = bf16(lo);
 *   q      = clamp(rint((w - bias) / scale), 0, 2^bits - 1), or 0 when the
 *            bf16 scale is 0.
 * The codes are integers decided by floating point, so they are decided in
 * the precision of the GPU kernel: binary32 with one rounding to nearest
 * even per operation (hi - lo, the division, w - bias, the quotient) and
 * rint ties to even; bf16 narrowing is to nearest even. Returns 0, or 1 on
 * bad arguments or a non-finite weight. */
int moe_ref_quantize(const float* w, int rows, int cols, int bits, int group,
                     uint8_t* codes, uint16_t* scale, uint16_t* bias) {
  if (!w || !codes || !scale || !bias) return 1;
  if (!pack_args_ok(rows, cols, bits, group)) return 1;
  int ng = cols / group;
  float levels = (float)((1 << bits) - 1);
  for (int r = 0; r < rows; ++r) {
    for (int g = 0; g < ng; ++g) {
      const float* wg = w + (size_t)r * cols + (size_t)g * group;
      float lo = wg[0], hi = wg[0];
      for (int j = 0; j < group; ++j) {
        if (!isfinite(wg[j])) return 1;
        if (wg[j] < lo) lo = wg[j];
        if (wg[j] > hi) hi = wg[j];
      }
      float range = hi - lo;
      float s32 = range / levels;
      uint16_t sbits = moe_ref_f64_to_bf16((double)s32);
      uint16_t bbits = moe_ref_f64_to_bf16((double)lo);
      float sf = (float)moe_ref_bf16_to_f64(sbits);
      float bf = (float)moe_ref_bf16_to_f64(bbits);
      size_t rg = (size_t)r * ng + g;
      scale[rg] = sbits;
      bias[rg] = bbits;
      for (int j = 0; j < group; ++j) {
        int q = 0;
        if (sf != 0.0f) {
          float d = wg[j] - bf;
          float t = d / sf;
          float qr = rintf(t);
          q = qr < 0.0f ? 0 : (qr > levels ? (int)levels : (int)qr);
        }
        codes[(size_t)r * cols + (size_t)g * group + j] = (uint8_t)q;
      }
    }
  }
  return 0;
}

/* ---- dequant mat-vec --------------------------------------------------- */

/* Plain definition: dequantise each weight, w = q*scale + bias, then dot. */
void moe_ref_dequant_gemv(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                          int rows, int cols, int group, const double* x, double* y) {
  int ng = cols / group;
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) {
      double s = moe_ref_bf16_to_f64(scale[(size_t)r * ng + c / group]);
      double b = moe_ref_bf16_to_f64(bias[(size_t)r * ng + c / group]);
      double w = (double)codes[(size_t)r * cols + c] * s + b;
      acc += w * x[c];
    }
    y[r] = acc;
  }
}

/* The Flash-MoE page's rearrangement (section "Kernel dequant toi uu FMA"):
 * (q*scale + bias)*x  ==  fma(q, scale*x, bias*x). */
void moe_ref_dequant_gemv_fma(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                              int rows, int cols, int group, const double* x, double* y) {
  int ng = cols / group;
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) {
      double s = moe_ref_bf16_to_f64(scale[(size_t)r * ng + c / group]);
      double b = moe_ref_bf16_to_f64(bias[(size_t)r * ng + c / group]);
      acc += fma((double)codes[(size_t)r * cols + c], s * x[c], b * x[c]);
    }
    y[r] = acc;
  }
}

/* The same sum taken group by group: scale * sum(q*x) + bias * sum(x). */
void moe_ref_dequant_gemv_grouped(const uint8_t* codes, const uint16_t* scale, const uint16_t* bias,
                                  int rows, int cols, int group, const double* x, double* y) {
  int ng = cols / group;
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int g = 0; g < ng; ++g) {
      double qx = 0.0, xs = 0.0;
      for (int j = 0; j < group; ++j) {
        int c = g * group + j;
        qx += (double)codes[(size_t)r * cols + c] * x[c];
        xs += x[c];
      }
      acc += moe_ref_bf16_to_f64(scale[(size_t)r * ng + g]) * qx +
             moe_ref_bf16_to_f64(bias[(size_t)r * ng + g]) * xs;
    }
    y[r] = acc;
  }
}

/* ---- router: logits, softmax, top-K ----------------------------------- */

void moe_ref_router_logits(const uint16_t* x_bf16, const uint16_t* wr_bf16, int H, int E, double* logits) {
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h)
      acc += moe_ref_bf16_to_f64(wr_bf16[(size_t)e * H + h]) * moe_ref_bf16_to_f64(x_bf16[h]);
    logits[e] = acc;
  }
}

void moe_ref_softmax(const double* logits, int E, double* p) {
  double m = logits[0];
  for (int e = 1; e < E; ++e)
    if (logits[e] > m) m = logits[e];
  double z = 0.0;
  for (int e = 0; e < E; ++e) {
    p[e] = exp(logits[e] - m);
    z += p[e];
  }
  for (int e = 0; e < E; ++e) p[e] /= z;
}

typedef struct {
  double logit;
  int index;
} ranked;

/* larger logit first; equal logits: lower expert index first */
static int by_rank(const void* pa, const void* pb) {
  const ranked* a = (const ranked*)pa;
  const ranked* b = (const ranked*)pb;
  if (a->logit > b->logit) return -1;
  if (a->logit < b->logit) return 1;
  return (a->index > b->index) - (a->index < b->index);
}

int moe_ref_topk(const double* logits, int E, int K, int renorm, const int32_t* forced,
                 int32_t* idx, double* w) {
  if (E <= 0 || K <= 0 || K > E) return 1;
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  if (!p) return 1;
  moe_ref_softmax(logits, E, p);
  if (forced) {
    for (int k = 0; k < K; ++k) {
      if (forced[k] < 0 || forced[k] >= E) {
        free(p);
        return 1;
      }
      idx[k] = forced[k];
    }
  } else {
    ranked* all = (ranked*)malloc(sizeof(ranked) * (size_t)E);
    if (!all) {
      free(p);
      return 1;
    }
    for (int e = 0; e < E; ++e) {
      all[e].logit = logits[e];
      all[e].index = e;
    }
    qsort(all, (size_t)E, sizeof(ranked), by_rank);
    for (int k = 0; k < K; ++k) idx[k] = all[k].index;
    free(all);
  }
  double total = 0.0;
  for (int k = 0; k < K; ++k) {
    w[k] = p[idx[k]];
    total += w[k];
  }
  if (renorm)
    for (int k = 0; k < K; ++k) w[k] /= total;
  free(p);
  return 0;
}

/* ---- SwiGLU, expert FFN ----------------------------------------------- */

double moe_ref_silu(double z) { return z / (1.0 + exp(-z)); }

void moe_ref_swiglu(const double* g, const double* u, int n, double* h) {
  for (int i = 0; i < n; ++i) h[i] = moe_ref_silu(g[i]) * u[i];
}

void moe_ref_expert_ffn(int H, int I, int group,
                        const uint8_t* codes_g, const uint16_t* scale_g, const uint16_t* bias_g,
                        const uint8_t* codes_u, const uint16_t* scale_u, const uint16_t* bias_u,
                        const uint8_t* codes_d, const uint16_t* scale_d, const uint16_t* bias_d,
                        const double* x, double* y) {
  double* g = (double*)malloc(sizeof(double) * (size_t)I);
  double* u = (double*)malloc(sizeof(double) * (size_t)I);
  double* h = (double*)malloc(sizeof(double) * (size_t)I);
  if (!g || !u || !h) {
    free(g);
    free(u);
    free(h);
    for (int i = 0; i < H; ++i) y[i] = NAN;
    return;
  }
  moe_ref_dequant_gemv(codes_g, scale_g, bias_g, I, H, group, x, g);
  moe_ref_dequant_gemv(codes_u, scale_u, bias_u, I, H, group, x, u);
  moe_ref_swiglu(g, u, I, h);
  moe_ref_dequant_gemv(codes_d, scale_d, bias_d, H, I, group, h, y);
  free(g);
  free(u);
  free(h);
}

/* ---- combine, shared gate, RMSNorm ------------------------------------ */

double moe_ref_shared_gate(const uint16_t* wsg_bf16, const uint16_t* x_bf16, int H) {
  double a = 0.0;
  for (int h = 0; h < H; ++h) a += moe_ref_bf16_to_f64(wsg_bf16[h]) * moe_ref_bf16_to_f64(x_bf16[h]);
  return 1.0 / (1.0 + exp(-a));
}

void moe_ref_combine(int H, int K, const double* y, const double* w, double gamma,
                     const double* r, double* out) {
  for (int i = 0; i < H; ++i) {
    double acc = r[i];
    for (int k = 0; k < K; ++k) acc += w[k] * y[(size_t)k * H + i];
    acc += gamma * y[(size_t)K * H + i];
    out[i] = acc;
  }
}

void moe_ref_rmsnorm(const double* v, int H, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < H; ++i) ss += v[i] * v[i];
  double inv = 1.0 / sqrt(ss / H + eps);
  for (int i = 0; i < H; ++i) out[i] = v[i] * inv;
}

void moe_ref_rmsnorm_bf16(const double* v, int H, double eps, uint16_t* out) {
  double* t = (double*)malloc(sizeof(double) * (size_t)H);
  if (!t) return;
  moe_ref_rmsnorm(v, H, eps, t);
  for (int i = 0; i < H; ++i) out[i] = moe_ref_f64_to_bf16(t[i]);
  free(t);
}

/* The RMS norm as a kernel of its own (Flash-MoE page, "Metal Compute
 * Shaders"), with a per-element bf16 weight: out[i] = bf16(v[i] * inv * w[i]),
 * inv = 1 / sqrt(mean(v^2) + eps), in fp64, rounded once to nearest-even
 * bf16. w == NULL means unit weight. */
void moe_ref_rmsnorm_weighted_bf16(const double* v, const uint16_t* w, int H, double eps, uint16_t* out) {
  double ss = 0.0;
  for (int i = 0; i < H; ++i) ss += v[i] * v[i];
  double inv = 1.0 / sqrt(ss / H + eps);
  for (int i = 0; i < H; ++i) {
    double wi = w ? moe_ref_bf16_to_f64(w[i]) : 1.0;
    out[i] = moe_ref_f64_to_bf16(v[i] * inv * wi);
  }
}
