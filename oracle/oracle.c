/*
 * oracle.c -- plain double-precision CPU oracle of the Flash-MoE per-layer
 * mixture-of-experts decode step.  TEST INFRASTRUCTURE ONLY (see oracle.h).
 *
 * Every function is the textbook definition of its step, written out with no
 * blocking, fusion or reordering beyond an OpenMP split of independent output
 * rows.  Where the pages leave a step open the reading taken is stated at the
 * function.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define GROUP 64

double orc_bf16_value(uint16_t v) {
  uint32_t u = (uint32_t)v << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round to the bf16 grid: quantum 2^(e-7) for a value with binary exponent e
 * (8 significant bits), 2^-133 below the normal range; nearbyint rounds ties to
 * even in the default rounding mode.  The rounded value is exactly a float. */
uint16_t orc_round_bf16(double v) {
  if (v != v) return 0x7FC0;
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  if (isinf(v)) return v > 0 ? 0x7F80 : 0xFF80;
  int e = ilogb(v);
  int qexp = e < -126 ? -133 : e - 7;
  double q = nearbyint(ldexp(v, -qexp));
  double r = ldexp(q, qexp);
  if (fabs(r) >= ldexp(1.0, 128)) return v > 0 ? 0x7F80 : 0xFF80;
  float f = (float)r; /* exact: r has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

static void matrix_shape(int hidden, int inter, int m, int64_t* R, int64_t* C) {
  if (m < 2) { *R = inter; *C = hidden; }
  else { *R = hidden; *C = inter; }
}

static int64_t matrix_bytes(int hidden, int inter, int bits, int m) {
  int64_t R, C;
  matrix_shape(hidden, inter, m, &R, &C);
  return R * C * bits / 8 + 2 * 2 * R * (C / GROUP);
}

/* "Flash-MoE: Running a 400 Billion Parameter Model on a MacBook",
 * section "The Architecture", sizes one 4-bit expert at about
 * 6.75 MB; three matrices of 4096 x 1024 codes plus a bf16 scale and bias per 64 codes give
 * exactly 7,077,888 bytes = 6.75 MiB. */
int64_t orc_blob_bytes(int hidden, int inter, int bits) {
  return matrix_bytes(hidden, inter, bits, 0) + matrix_bytes(hidden, inter, bits, 1) +
         matrix_bytes(hidden, inter, bits, 2);
}

/* Dequantisation, w = q * scale + bias with one bf16 (scale, bias) per group of
 * 64 consecutive columns of a row ("Flash-MoE: Running a 400 Billion Parameter Model on a MacBook",
 * section "The Architecture": the inner
 * loop dequantises with fused multiply-adds; the affine form, group size and
 * dtypes are readings taken where the pages are silent).  Code c of row r is field c % (32/bits) of little-endian 32-bit
 * word c / (32/bits) of that row. */
double orc_weight(const uint8_t* blob, int hidden, int inter, int bits, int m, int r, int c) {
  int64_t off = 0;
  for (int j = 0; j < m; ++j) off += matrix_bytes(hidden, inter, bits, j);
  int64_t R, C;
  matrix_shape(hidden, inter, m, &R, &C);
  const uint8_t* codes = blob + off;
  int per_word = 32 / bits;
  int64_t word_index = (int64_t)r * (C / per_word) + c / per_word;
  uint32_t word;
  memcpy(&word, codes + 4 * word_index, 4);
  uint32_t q = (word >> (bits * (c % per_word))) & ((1u << bits) - 1u);
  int64_t ng = C / GROUP;
  const uint8_t* scales = codes + R * C * bits / 8;
  const uint8_t* biases = scales + 2 * R * ng;
  uint16_t s16, b16;
  memcpy(&s16, scales + 2 * ((int64_t)r * ng + c / GROUP), 2);
  memcpy(&b16, biases + 2 * ((int64_t)r * ng + c / GROUP), 2);
  return orc_bf16_value(s16) * (double)q + orc_bf16_value(b16);
}

/* RMSNorm ahead of the mixture-of-experts block (the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works":
 * the second command buffer normalises before it routes; the epsilon is the
 * reading taken where the pages are silent). */
void orc_rmsnorm(const uint16_t* h, const uint16_t* w, int hidden, double eps, uint16_t* z) {
  double ss = 0.0;
  for (int i = 0; i < hidden; ++i) {
    double v = orc_bf16_value(h[i]);
    ss += v * v;
  }
  double r = 1.0 / sqrt(ss / (double)hidden + eps);
  for (int i = 0; i < hidden; ++i) {
    double wi = w ? orc_bf16_value(w[i]) : 1.0;
    z[i] = orc_round_bf16(orc_bf16_value(h[i]) * r * wi);
  }
}

/* Router GEMV, hidden -> one logit per expert (the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works":
 * the second command buffer computes the routing; the themata summary "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * Key Takeaways:
 * 512 experts per layer). */
void orc_router_logits(const uint16_t* wr, const float* bias, const uint16_t* z, int hidden, int n_experts,
                       float* logits) {
#pragma omp parallel for schedule(static)
  for (int e = 0; e < n_experts; ++e) {
    double d = 0.0;
    for (int h = 0; h < hidden; ++h) d += orc_bf16_value(wr[(int64_t)e * hidden + h]) * orc_bf16_value(z[h]);
    if (bias) d += (double)bias[e];
    logits[e] = (float)d;
  }
}

typedef struct { double p; double l; int e; } prob_entry;

/* larger probability first; equal probabilities (exact ties, or both rounded
 * to 0) by larger logit, then lower expert index */
static int by_prob_desc(const void* a, const void* b) {
  const prob_entry* x = (const prob_entry*)a;
  const prob_entry* y = (const prob_entry*)b;
  if (x->p > y->p) return -1;
  if (x->p < y->p) return 1;
  if (x->l > y->l) return -1;
  if (x->l < y->l) return 1;
  return (x->e > y->e) - (x->e < y->e);
}

/* Softmax and top-K (the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works":
 * the host takes the softmax and picks the top K; the themata summary "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * Key Takeaways: K = 4).
 * Renormalising the K selected probabilities is a reading taken where the pages are silent.
 * Non-finite logits, where the pages are silent too: a NaN logit counts as
 * -inf, and when the largest logit is infinite the softmax is its limit, the
 * whole mass shared equally by the experts whose logit equals the largest
 * (all of them when every logit is -inf). */
void orc_topk(const float* logits, int n_experts, int top_k, int32_t* idx, double* w, double* p) {
  prob_entry* ent = (prob_entry*)malloc(sizeof(prob_entry) * (size_t)n_experts);
  double mx = -INFINITY;
  for (int e = 0; e < n_experts; ++e) {
    ent[e].l = isnan(logits[e]) ? -INFINITY : (double)logits[e];
    ent[e].e = e;
    mx = fmax(mx, ent[e].l);
  }
  double denom = 0.0;
  for (int e = 0; e < n_experts; ++e) {
    if (isinf(mx))
      ent[e].p = ent[e].l == mx ? 1.0 : 0.0;
    else
      ent[e].p = exp(ent[e].l - mx);
    denom += ent[e].p;
  }
  for (int e = 0; e < n_experts; ++e) {
    ent[e].p /= denom;
    if (p) p[e] = ent[e].p;
  }
  qsort(ent, (size_t)n_experts, sizeof(prob_entry), by_prob_desc);
  double sel = 0.0;
  for (int k = 0; k < top_k; ++k) sel += ent[k].p;
  for (int k = 0; k < top_k; ++k) {
    idx[k] = ent[k].e;
    w[k] = ent[k].p / sel;
  }
  free(ent);
}

/* SwiGLU expert feed-forward with inline dequantisation (the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works":
 * the third command buffer runs the experts; "Flash-MoE: Running a 400 Billion Parameter Model on a MacBook",
 * section "The Architecture":
 * dequantisation fused into the multiply-adds).  silu(t) = t/(1+e^-t) applied
 * to the gate projection, times the up projection, is the reading taken of
 * the activation. */
void orc_expert(const uint8_t* blob, int hidden, int inter, int bits, const uint16_t* z, double* g, double* u,
                double* a, double* y) {
  double* gg = (double*)malloc(sizeof(double) * (size_t)inter);
  double* uu = (double*)malloc(sizeof(double) * (size_t)inter);
  double* aa = (double*)malloc(sizeof(double) * (size_t)inter);
#pragma omp parallel for schedule(static)
  for (int r = 0; r < inter; ++r) {
    double sg = 0.0, su = 0.0;
    for (int c = 0; c < hidden; ++c) {
      double x = orc_bf16_value(z[c]);
      sg += orc_weight(blob, hidden, inter, bits, 0, r, c) * x;
      su += orc_weight(blob, hidden, inter, bits, 1, r, c) * x;
    }
    gg[r] = sg;
    uu[r] = su;
    aa[r] = sg / (1.0 + exp(-sg)) * su;
  }
#pragma omp parallel for schedule(static)
  for (int j = 0; j < hidden; ++j) {
    double s = 0.0;
    for (int r = 0; r < inter; ++r) s += orc_weight(blob, hidden, inter, bits, 2, j, r) * aa[r];
    y[j] = s;
  }
  if (g) memcpy(g, gg, sizeof(double) * (size_t)inter);
  if (u) memcpy(u, uu, sizeof(double) * (size_t)inter);
  if (a) memcpy(a, aa, sizeof(double) * (size_t)inter);
  free(gg);
  free(uu);
  free(aa);
}

/* Weighted combine into the residual (the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works":
 * the third command buffer also combines the expert outputs); the shared expert
 * that the same section adds to the K routed ones enters with weight 1. */
void orc_combine(const uint16_t* h, const double* w, const double* y_routed, const double* y_shared, int hidden,
                 int top_k, double* out_f64, uint16_t* out) {
  for (int j = 0; j < hidden; ++j) {
    double s = orc_bf16_value(h[j]);
    for (int k = 0; k < top_k; ++k) s += w[k] * y_routed[(int64_t)k * hidden + j];
    s += y_shared[j];
    if (out_f64) out_f64[j] = s;
    if (out) out[j] = orc_round_bf16(s);
  }
}

/* 4-bit -> 2-bit requantisation of one canonical expert blob.  The page
 * "Flash-MoE Inference Engine", section "Weight Preparation" (step 3, optional
 * 2-bit requantisation), converts the 4-bit expert files to 2-bit with a script
 * but gives no algorithm.  Reading taken: every 64-column group of every row is
 * refitted on its own with an affine grid spanning the group's smallest and
 * largest dequantised weight, each step one IEEE fp32 operation rounded to
 * nearest even (so that the integer codes are decided with the same arithmetic
 * by any implementation):
 *   w_c  = fmaf(q4_c, s4, b4)          s4, b4: the group's bf16 scale and bias
 *   lo   = min_c w_c,  hi = max_c w_c
 *   s2   = bf16((hi - lo) / 3)
 *   b2   = bf16(lo)
 *   inv  = s2 > 0 ? 1 / s2 : 0
 *   q2_c = min(max(rint((w_c - b2) * inv), 0), 3)
 * The output is the canonical 2-bit blob of the same matrices. */
void orc_requant_4to2(const uint8_t* src, int hidden, int inter, uint8_t* dst) {
  int64_t in_off = 0, out_off = 0;
  for (int m = 0; m < 3; ++m) {
    int64_t R, C;
    matrix_shape(hidden, inter, m, &R, &C);
    const int64_t ng = C / GROUP;
    const uint8_t* in_codes = src + in_off;
    const uint8_t* in_s = in_codes + R * C / 2;
    const uint8_t* in_b = in_s + 2 * R * ng;
    uint8_t* out_codes = dst + out_off;
    uint8_t* out_s = out_codes + R * C / 4;
    uint8_t* out_b = out_s + 2 * R * ng;
    for (int64_t r = 0; r < R; ++r) {
      for (int64_t g = 0; g < ng; ++g) {
        uint16_t s16, b16;
        memcpy(&s16, in_s + 2 * (r * ng + g), 2);
        memcpy(&b16, in_b + 2 * (r * ng + g), 2);
        const float s4 = (float)orc_bf16_value(s16), b4 = (float)orc_bf16_value(b16);
        float w[GROUP];
        for (int c = 0; c < GROUP; ++c) {
          const int64_t col = g * GROUP + c;
          uint32_t word;
          memcpy(&word, in_codes + 4 * ((r * C + col) / 8), 4);
          const uint32_t q = (word >> (4 * (col % 8))) & 15u;
          w[c] = fmaf((float)q, s4, b4);
        }
        float lo = w[0], hi = w[0];
        for (int c = 1; c < GROUP; ++c) {
          if (w[c] < lo) lo = w[c];
          if (w[c] > hi) hi = w[c];
        }
        const float span = hi - lo;
        const float third = span / 3.0f;
        const uint16_t s2b = orc_round_bf16((double)third);
        const uint16_t b2b = orc_round_bf16((double)lo);
        const float s2 = (float)orc_bf16_value(s2b), b2 = (float)orc_bf16_value(b2b);
        const float inv = s2 > 0.0f ? 1.0f / s2 : 0.0f;
        memcpy(out_s + 2 * (r * ng + g), &s2b, 2);
        memcpy(out_b + 2 * (r * ng + g), &b2b, 2);
        for (int c = 0; c < GROUP; c += 16) {
          uint32_t word = 0;
          for (int k = 0; k < 16; ++k) {
            const float d = w[c + k] - b2;
            const float t = d * inv;
            float qf = rintf(t);
            if (qf < 0.0f) qf = 0.0f;
            if (qf > 3.0f) qf = 3.0f;
            word |= (uint32_t)qf << (2 * k);
          }
          memcpy(out_codes + 4 * ((r * C + g * GROUP + c) / 16), &word, 4);
        }
      }
    }
    in_off += matrix_bytes(hidden, inter, 4, m);
    out_off += matrix_bytes(hidden, inter, 2, m);
  }
}
