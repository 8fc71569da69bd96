/*
 * oracle.h -- plain, slow, double-precision CPU oracle of the Flash-MoE
 * per-layer mixture-of-experts decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code with the CUDA
 * library; both only read the same canonical expert blobs produced by the
 * seeded generator.
 *
 * What it computes (pages: the wiki page "Flash-MoE", Technical Architecture;
 * the Hysen Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop",
 * section "How the SSD expert streaming pipeline works"; "Flash-MoE: Running a
 * 400 Billion Parameter Model on a MacBook", section "The Architecture"):
 * per token and layer, optional RMSNorm of the layer input, router GEMV over
 * E experts, softmax, top-K selection with the selected probabilities
 * renormalised, SwiGLU feed-forward of the K selected experts and of one shared
 * expert with weights dequantised as w = q*scale + bias (one bf16 scale and bias
 * per 64 consecutive inputs of a row), and the weighted combine into the
 * residual.  Rounding points mirrored from the CUDA library's contract: z is
 * stored as bf16, router logits as fp32, the layer output as bf16; everything
 * else is exact double arithmetic.
 */
#ifndef FMOE_ORACLE_H
#define FMOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exact value of a bf16 bit pattern. */
double orc_bf16_value(uint16_t v);
/* Nearest bf16 to v, ties to even. */
uint16_t orc_round_bf16(double v);
/* Size in bytes of one canonical expert blob. */
int64_t orc_blob_bytes(int hidden, int inter, int bits);
/* Dequantised weight of matrix m (0 gate [I][H], 1 up [I][H], 2 down [H][I]). */
double orc_weight(const uint8_t* blob, int hidden, int inter, int bits, int m, int r, int c);
/* 4-bit -> 2-bit requantisation of one canonical expert blob: per 64-group an
 * affine min/max refit decided in IEEE fp32 (steps at the definition). */
void orc_requant_4to2(const uint8_t* src, int hidden, int inter, uint8_t* dst);
/* z = bf16(h / sqrt(mean(h^2) + eps) * w); w may be NULL (treated as 1). */
void orc_rmsnorm(const uint16_t* h, const uint16_t* w, int hidden, double eps, uint16_t* z);
/* Router logits, fp32-rounded: logits[e] = fp32(sum_h Wr[e][h] z[h] + bias[e]). */
void orc_router_logits(const uint16_t* wr, const float* bias, const uint16_t* z, int hidden, int n_experts,
                       float* logits);
/* Softmax over all experts, then the K largest (ties: lower index first), then
 * w_k = p[idx_k] / sum_j p[idx_j].  p (optional) receives the full softmax. */
void orc_topk(const float* logits, int n_experts, int top_k, int32_t* idx, double* w, double* p);
/* One expert's SwiGLU: g = Wg z, u = Wu z, a = silu(g) u, y = Wd a.  g, u, a are
 * optional outputs of length inter; y has length hidden. */
void orc_expert(const uint8_t* blob, int hidden, int inter, int bits, const uint16_t* z, double* g,
                double* u, double* a, double* y);
/* out = h + sum_k w[k] * y_routed[k] + y_shared, returned exact (out_f64,
 * optional) and rounded to bf16 (out). y_routed is [top_k][hidden]. */
void orc_combine(const uint16_t* h, const double* w, const double* y_routed, const double* y_shared, int hidden,
                 int top_k, double* out_f64, uint16_t* out);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_ORACLE_H */
